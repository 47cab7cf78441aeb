"""Caller-supplied buffers in the Python binding.

Every output a caller passes (out, packed, scales, codes, block_scales,
global_scale) must have the output's dtype and element count, be
contiguous and sit on the device the call runs on, or on the host; status
and workspace words must be device tensors.  Anything else is rejected
before a kernel is launched, so that no kernel writes outside a buffer.
A host output receives the result by a copy after the call.

The helper checks run on the CPU; the end-to-end cases need the GPU.
"""
import numpy as np
import pytest
import torch

import nvfp4_quantization_amax_b200 as mxq
from nvfp4_quantization_amax_b200 import _abi
import oracle
import synthetic as gen

CPU = torch.device("cpu")


# ------------------------------------------------------------ host logic

def test_out_allocates_when_none():
    buf, target = _abi._out(None, (3, 4), torch.uint8, CPU, "x")
    assert tuple(buf.shape) == (3, 4) and buf.dtype == torch.uint8 and target is None


def test_out_rejects_wrong_dtype():
    with pytest.raises(TypeError, match="packed must be torch.uint8"):
        _abi._out(torch.empty(12, dtype=torch.int8), (3, 4), torch.uint8, CPU, "packed")


def test_out_rejects_wrong_element_count():
    with pytest.raises(ValueError, match="must hold 12 elements"):
        _abi._out(torch.empty(11, dtype=torch.uint8), (3, 4), torch.uint8, CPU, "out")
    with pytest.raises(ValueError, match="must hold 12 elements"):
        _abi._out(torch.empty(13, dtype=torch.uint8), (3, 4), torch.uint8, CPU, "out")


def test_out_rejects_non_contiguous():
    t = torch.empty(4, 6, dtype=torch.uint8)[:, ::2]
    assert t.numel() == 12
    with pytest.raises(ValueError, match="contiguous"):
        _abi._out(t, (3, 4), torch.uint8, CPU, "out")


def test_out_accepts_any_shape_with_the_element_count():
    t = torch.empty(2, 6, dtype=torch.uint8)
    buf, target = _abi._out(t, (3, 4), torch.uint8, CPU, "out")
    # a host buffer: the call computes into a fresh buffer viewed like it
    assert target is t and tuple(buf.shape) == (2, 6) and buf.data_ptr() != t.data_ptr()


def test_device_word_rules():
    assert _abi._device_word(None, torch.int32, 1, CPU, "status").value is None
    with pytest.raises(ValueError, match="status must be a tensor on"):
        _abi._device_word(torch.zeros(1, dtype=torch.int32), torch.int32, 1,
                          torch.device("cuda", 0), "status")


# ------------------------------------------------------------ on the GPU

DEV = "cuda"


@pytest.mark.gpu
def test_wrong_outputs_raise_before_any_launch():
    x = gen.normal_bf16(11, (8, 256), device=DEV)
    guard = torch.full((8, 127), 0x5A, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        mxq.mx_quantize(x, guard, None)
    with pytest.raises(ValueError):
        mxq.quantize_cache(x, "nvfp4", 16, torch.empty(8, 255, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(TypeError):
        mxq.mx_dequantize(*mxq.mx_quantize(x), torch.bfloat16,
                          torch.empty(8, 256, dtype=torch.float16, device=DEV))
    with pytest.raises(ValueError):
        mxq.nvfp4_quantize(x, workspace=torch.empty(8, dtype=torch.uint8, device=DEV))
    with pytest.raises(ValueError):
        mxq.nvfp4_quantize(x, global_scale=torch.empty(2, dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    assert bool((guard == 0x5A).all())


@pytest.mark.gpu
def test_host_status_word_is_rejected():
    E, N, K, T = 2, 128, 256, 64
    a = gen.normal_bf16(12, (T, K), device=DEV)
    p, s = mxq.mx_quantize(gen.normal_bf16(13, (E, N, K), std=0.02, device=DEV))
    offs = torch.tensor([32, 64], dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError, match="status"):
        mxq.mxfp4_grouped_mm(a, p, s, offs, status=torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="x_packed"):
        mxq.w4a4_grouped_mm(a, p, s, offs, x_packed=torch.empty(T, K // 2, dtype=torch.uint8))


@pytest.mark.gpu
@pytest.mark.parametrize("pinned", [True, False])
def test_host_outputs_receive_the_result(pinned):
    x = gen.normal_bf16(14, (64, 512), device=DEV)
    want_p, want_s = mxq.mx_quantize(x)
    hp = torch.empty(64, 256, dtype=torch.uint8, pin_memory=pinned)
    hs = torch.empty(64, 16, dtype=torch.uint8, pin_memory=pinned)
    got_p, got_s = mxq.mx_quantize(x.cpu(), hp, hs)
    assert got_p is hp and got_s is hs
    assert torch.equal(hp, want_p.cpu()) and torch.equal(hs, want_s.cpu())

    out = torch.empty(64, 512, dtype=torch.bfloat16, pin_memory=pinned)
    y = mxq.mx_dequantize(hp, hs, torch.bfloat16, out)
    assert y is out and torch.equal(out, mxq.mx_dequantize(want_p, want_s).cpu())

    q = torch.empty(64, 512, dtype=torch.bfloat16, pin_memory=pinned)
    assert mxq.quantize_cache(x, "fp8", 128, q) is q
    assert torch.equal(q, mxq.quantize_cache(x, "fp8", 128).cpu())


@pytest.mark.gpu
def test_host_outputs_match_the_oracle():
    x = gen.normal_bf16(15, (32, 256), device="cpu")
    packed = torch.empty(32, 128, dtype=torch.uint8, pin_memory=True)
    scales = torch.empty(32, 8, dtype=torch.uint8, pin_memory=True)
    mxq.mx_quantize(x, packed, scales)
    wp, ws = oracle.mx_quantize(x.view(torch.int16).numpy().view(np.uint16), "bf16")
    assert np.array_equal(packed.numpy(), np.asarray(wp, dtype=np.uint8).reshape(32, 128))
    assert np.array_equal(scales.numpy(), np.asarray(ws, dtype=np.uint8).reshape(32, 8))


@pytest.fixture
def small_chunks():
    # stream host tensors in many small chunks (ragged last one included)
    old = _abi.HOST_CHUNK_BYTES
    _abi.HOST_CHUNK_BYTES = 3000
    yield
    _abi.HOST_CHUNK_BYTES = old


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_streamed_host_calls_equal_whole_device_calls(small_chunks, dtype):
    x = gen.mixed_blocks(37, 256, device=DEV).to(dtype)  # 37 rows: chunks of 5 or 2 rows
    hx = x.cpu().pin_memory()
    p, s = mxq.mx_quantize(x)
    hp, hs = mxq.mx_quantize(hx)
    assert not hp.is_cuda and torch.equal(hp, p.cpu()) and torch.equal(hs, s.cpu())
    y = mxq.mx_dequantize(p, s, dtype)
    hy = mxq.mx_dequantize(hp.pin_memory(), hs.pin_memory(), dtype)
    assert torch.equal(hy.view(torch.uint8), y.cpu().view(torch.uint8))
    for fmt, B in (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)):
        q = mxq.quantize_cache(x, fmt, B)
        hq = mxq.quantize_cache(hx, fmt, B)
        assert torch.equal(hq.view(torch.uint8), q.cpu().view(torch.uint8)), fmt


@pytest.mark.gpu
def test_streamed_host_calls_fill_caller_buffers_and_report_errors(small_chunks):
    hx = gen.normal_bf16(16, (40, 64)).pin_memory()
    hp = torch.empty(40, 32, dtype=torch.uint8)                # pageable target
    hs = torch.empty(40, 2, dtype=torch.uint8, pin_memory=True)
    rp, rs = mxq.mx_quantize(hx, hp, hs)
    assert rp is hp and rs is hs
    wp, ws = mxq.mx_quantize(hx.to(DEV))
    assert torch.equal(hp, wp.cpu()) and torch.equal(hs, ws.cpu())
    with pytest.raises(mxq.MxqError):
        mxq.quantize_cache(hx, "fp8", 0)  # block_size < 1, reported by the first chunk


@pytest.mark.gpu
def test_streamed_packed_cache_and_nvfp4_dequant_equal_device_calls(small_chunks):
    x = gen.mixed_blocks(29, 256, device=DEV)
    hx = x.cpu().pin_memory()
    for fmt, B in (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)):
        c, s = mxq.quantize_cache_packed(x, fmt, B)
        hc, hs = mxq.quantize_cache_packed(hx, fmt, B)
        assert torch.equal(hc, c.cpu()) and torch.equal(hs, s.cpu()), fmt
        y = mxq.dequantize_cache_packed(c, s, fmt, B)
        hy = mxq.dequantize_cache_packed(hc.pin_memory(), hs.pin_memory(), fmt, B)
        assert torch.equal(hy.view(torch.uint8), y.cpu().view(torch.uint8)), fmt
    p, s, g = mxq.nvfp4_quantize(x)
    y = mxq.nvfp4_dequantize(p, s, g, torch.float32)
    hy = mxq.nvfp4_dequantize(p.cpu().pin_memory(), s.cpu().pin_memory(), g.cpu(), torch.float32)
    assert not hy.is_cuda and torch.equal(hy.view(torch.uint8), y.cpu().view(torch.uint8))


def test_prequantized_w4a4_operands_must_be_cuda_tensors():
    # refused on the host, before any library call
    p = torch.zeros(2, 128, 128, dtype=torch.uint8)
    s = torch.zeros(2, 128, 8, dtype=torch.uint8)
    offs = torch.tensor([32, 64], dtype=torch.int32)
    xq = torch.zeros(64, 128, dtype=torch.uint8)
    xs = torch.zeros(64, 8, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        mxq.w4a4_grouped_mm(None, p, s, offs, x_quantized=(xq, xs))
    with pytest.raises(ValueError, match="CUDA"):
        mxq.nvfp4_w4a4_grouped_mm(None, p, torch.zeros(2, 128, 16, dtype=torch.uint8),
                                  torch.ones(2), offs,
                                  x_quantized=(xq, torch.zeros(64, 16, dtype=torch.uint8),
                                               torch.ones(1)))

