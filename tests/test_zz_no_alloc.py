"""The allocation-free NVFP4 entry point, called through the C ABI.

nvfp4_quantize_noalloc serves callers that may not allocate device memory
while they run (their memory pool is fixed up front, and cudaMalloc would
synchronize or fail); it takes its 16 bytes of scratch from a static device
array inside the library instead of a caller workspace.  This test checks
that it returns exactly what the workspace entry point returns, on two calls
in a row: the first input has the larger maximum, so a scratch word left over
from the first call would corrupt the second call's per-tensor scale.
"""
import ctypes

import pytest
import torch

import nvfp4_quantization_amax_b200 as mxq
import synthetic as gen

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L = mxq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    inputs = [gen.kv_cache((1, 256, 512), device=dev).view(256, 512),  # max ~1e4
              gen.expert_weights(2, 512, 1024, device=dev).view(1024, 1024)]  # max ~0.1
    assert inputs[0].float().abs().max() > inputs[1].float().abs().max()
    for x in inputs:
        want_p, want_s, want_g = mxq.nvfp4_quantize(x)
        rows, K = x.shape
        p = torch.full_like(want_p, 0xAA)
        s = torch.full_like(want_s, 0xAA)
        g = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
        rc = L.nvfp4_quantize_noalloc(_p(x), 0, rows, K, _p(p), _p(s), _p(g), stream)
        assert rc == 0, mxq.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(g, want_g)
        assert torch.equal(s, want_s)
        assert torch.equal(p, want_p)
