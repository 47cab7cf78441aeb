"""Out-of-bounds write checks: canary padding around every output buffer.

Each output a call writes here sits inside a larger allocation whose 4 KiB
before and after hold a sentinel byte; after the call and a synchronize the
padding must be intact (no kernel wrote outside its buffer).  The shapes are
small and ragged: an odd row count, a tail channel group, experts without
tokens, and widths that take the general kernels as well as the streaming
and tensor-core ones.  Values are checked against the oracle elsewhere; this
file only guards the bounds.
"""
import math

import numpy as np
import pytest
import torch

import nvfp4_quantization_amax_b200 as mxq
import synthetic as gen

PAD = 4096
SENTINEL = 0xA5
DEV = "cuda"


class Padded:
    """A `shape` x `dtype` tensor `t` with PAD sentinel bytes on each side."""

    def __init__(self, shape, dtype, device=DEV):
        nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((PAD + nbytes + PAD,), SENTINEL, dtype=torch.uint8, device=device)
        self.t = self.raw[PAD:PAD + nbytes].view(dtype).view(shape)

    def intact(self):
        return bool((self.raw[:PAD] == SENTINEL).all()) and bool((self.raw[-PAD:] == SENTINEL).all())


def test_padding_helper_on_the_host():
    p = Padded((3, 5), torch.bfloat16, device="cpu")
    assert p.t.shape == (3, 5) and p.t.dtype == torch.bfloat16 and p.t.is_contiguous()
    assert p.t.data_ptr() - p.raw.data_ptr() == PAD
    p.t.fill_(1.0)
    assert p.intact()
    p.raw[PAD + 30] = 0  # one byte past the tensor
    assert not p.intact()
    q = Padded((1,), torch.int32, device="cpu")
    q.t.zero_()
    assert q.intact() and int(q.t.item()) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_streaming_calls_write_only_their_outputs(dtype):
    rows, K = 37, 224  # seven 32-blocks per row; 37 rows leave partial warps and waves
    x = gen.mixed_blocks(rows, K, device=DEV).to(dtype)
    bufs = []

    def pad(shape, dt):
        b = Padded(shape, dt)
        bufs.append(b)
        return b.t

    p, s = pad((rows, K // 2), torch.uint8), pad((rows, K // 32), torch.uint8)
    mxq.mx_quantize(x, p, s)
    mxq.mx_dequantize(p, s, dtype, pad((rows, K), dtype))
    # fast paths and general paths (tail group of 96, block sizes 24 and 14)
    for fmt, B in (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16), ("nvfp4", 24)):
        mxq.quantize_cache(x, fmt, B, pad((rows, K), dtype))
    for fmt, B in (("fp8", 32), ("fp8", 56), ("mxfp4", 32), ("mxfp4", 14), ("nvfp4", 16)):
        codes = pad((rows, K if fmt == "fp8" else K // 2), torch.uint8)
        sc = pad((rows, K // B), torch.uint8)
        mxq.quantize_cache_packed(x, fmt, B, codes, sc)
        mxq.dequantize_cache_packed(codes, sc, fmt, B, dtype, pad((rows, K), dtype))
    for rule in ("max", "mse"):
        np_, ns = pad((rows, K // 2), torch.uint8), pad((rows, K // 16), torch.uint8)
        g, ws = pad((1,), torch.float32), pad((16,), torch.uint8)
        mxq.nvfp4_quantize(x, np_, ns, g, ws, rule=rule)
        mxq.nvfp4_dequantize(np_, ns, g, dtype, pad((rows, K), dtype))
    torch.cuda.synchronize()
    assert all(b.intact() for b in bufs)


def _nv_weights(E, N, K, seed=41):
    packed = gen.random_bytes(E * N * (K // 2), gen.seed_for(seed, 1)).view(E, N, K // 2)
    u = gen.uniform(gen.seed_for(seed, 2), E * N * (K // 16))
    bs = (u * 17).floor().clamp_(max=16).to(torch.uint8).add_(0x30).view(E, N, K // 16)
    gw = torch.tensor([0.01 * (1 + e / E) for e in range(E)], dtype=torch.float32)
    return packed, bs, gw


@pytest.mark.gpu
@pytest.mark.parametrize("N,K", [(256, 512), (128, 192), (96, 96)])
def test_grouped_gemms_write_only_their_outputs(N, K):
    # (256, 512): CTA pairs both ways; (128, 192): one CTA forward, general
    # input gradient; (96, 96): general kernels
    counts = [37, 0, 61, 22]
    E, T = len(counts), sum(counts)
    offs = torch.tensor(np.cumsum(counts), dtype=torch.int32, device=DEV)
    packed, scales = gen.random_packed(E, N, K, 116, 124, workload=51)
    packed, scales = packed.to(DEV), scales.to(DEV)
    a = gen.normal_bf16(gen.seed_for(51, 3), (T, K), device=DEV)
    g = gen.normal_bf16(gen.seed_for(51, 4), (T, N), device=DEV)
    bufs = [Padded((T, N), torch.bfloat16), Padded((T, K), torch.bfloat16), Padded((1,), torch.int32)]
    y, gx, st = (b.t for b in bufs)
    st.zero_()
    mxq.mxfp4_grouped_mm(a, packed, scales, offs, False, y, st)
    mxq.mxfp4_grouped_mm(g, packed, scales, offs, True, gx, st)
    if K % 256 == 0 and N % 128 == 0:
        # W4A4 in MXFP4 (activation codes and scales padded too) and NVFP4
        more = [Padded((T, N), torch.bfloat16), Padded((T, K // 2), torch.uint8),
                Padded((T, K // 32), torch.uint8), Padded((T, N), torch.bfloat16)]
        bufs += more
        mxq.w4a4_grouped_mm(a, packed, scales, offs, more[0].t, st, more[1].t, more[2].t)
        nvp, nvs, nvg = (t.to(DEV) for t in _nv_weights(E, N, K))
        mxq.nvfp4_w4a4_grouped_mm(a, nvp, nvs, nvg, offs, more[3].t, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(b.intact() for b in bufs)
