"""GPU parity at the largest size the benchmark runs.

The bandwidth sweep's top point is the mixed-block workload x bf16
[2^21, 7168]: 15.0 G elements, 30 GB per bf16 tensor, so element indices pass
2^31 and byte offsets pass 2^32 inside one call.  Here the MXFP4 pack, the
unpack and the cache fake quantization in its three formats run on it in
whole-tensor calls, as the sweep times them, and the oracle checks sampled
rows: the first and the last, 16 seeded ones, and the rows around the places
where a 32-bit index or byte offset would wrap (element 2^31 of x and of the
bf16 outputs, byte 2^32 of the packed codes).  Inputs are those rows as the
GPU received them, copied back.  The NVFP4 max-rule quantize and unpack are
checked the same way at the size the benchmark times them, [64, 2048, 7168].
"""
import numpy as np
import pytest
import torch

import nvfp4_quantization_amax_b200 as mxq
import oracle
import synthetic as gen

pytestmark = pytest.mark.gpu

DEV = "cuda"
R, C = 1 << 21, 7168


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def _same(got, want, what):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got.reshape(-1) != want.reshape(-1))[0]
    assert bad.size == 0, "%s: %d mismatches, first at flat %s" % (what, bad.size, bad[:4])


def sampled_rows():
    wrap_elem = (1 << 31) // C         # holds element 2^31 (byte 2^32 of x and of the outputs)
    wrap_code = (1 << 32) // (C // 2)  # holds byte 2^32 of the packed codes
    rows = {0, R - 1}
    for w in (wrap_elem, wrap_code):
        rows |= {w - 1, w, w + 1}
    rng = np.random.default_rng(21)
    rows |= {int(r) for r in rng.choice(R, 16, replace=False)}
    return sorted(rows)


def test_streaming_kernels_at_the_largest_benchmark_size():
    torch.cuda.empty_cache()
    need = R * C * 2 * 2 + R * C // 2 + R * C // 32  # x, one output, codes, scales
    free, _ = torch.cuda.mem_get_info()
    if free < need + (8 << 30):
        pytest.skip("needs %.0f GB of free device memory, %.0f GB free" % (need / 1e9, free / 1e9))
    x = gen.mixed_blocks(R, C, device=DEV)
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((R, C // 32), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(x)
    rows = torch.tensor(sampled_rows(), device=DEV)
    xr = _bits(x[rows])

    mxq.mx_quantize(x, packed, scales)
    mxq.mx_dequantize(packed, scales, torch.bfloat16, out)
    want_p, want_s = oracle.mx_quantize(xr, "bf16")
    _same(_u8(packed[rows]), want_p, "packed rows")
    _same(_u8(scales[rows]), want_s, "scale rows")
    _same(_bits(out[rows]), oracle.mx_dequantize(want_p, want_s, "bf16"), "unpacked rows")
    assert int(scales.max()) < 255  # the pack never writes the E8M0 NaN byte

    for fmt, B in (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)):
        mxq.quantize_cache(x, fmt, B, out)
        _same(_bits(out[rows]), oracle.quantize_cache(xr, fmt, B), "%s B=%d rows" % (fmt, B))

    del x, packed, scales, out, rows
    torch.cuda.empty_cache()


def test_nvfp4_max_rule_at_the_benchmark_size():
    # NVFP4 quantize (max rule) and unpack of the expert weights bf16
    # [64, 2048, 7168], the size the benchmark times them at.  The per-tensor
    # scale needs max |x| over the whole tensor: taken on the host from every
    # element's magnitude bits (for finite bf16 they order like the values),
    # then the oracle gives g, and the codes, block scales and unpacked values
    # of the first, the last and 32 seeded rows.
    W = gen.expert_weights(device=DEV)
    p, s, g = mxq.nvfp4_quantize(W)
    y = mxq.nvfp4_dequantize(p, s, g)
    hb = _bits(W).reshape(-1, C)
    amax_bits = np.array([int((hb & 0x7FFF).max())], np.uint16)
    want_g = oracle.nvfp4_global_scale(oracle.decode(amax_bits, "bf16")[0])
    assert float(g.item()) == want_g
    n = hb.shape[0]
    seeded = np.random.default_rng(5).choice(n, 32, replace=False)
    rows = sorted({0, n - 1} | {int(r) for r in seeded})
    want_p, want_s = oracle.nvfp4_quantize_rows(hb[rows], want_g)
    idx = torch.tensor(rows, device=DEV)
    _same(_u8(p.view(-1, C // 2)[idx]), want_p, "packed rows")
    _same(_u8(s.view(-1, C // 16)[idx]), want_s, "block scale rows")
    _same(_bits(y.view(-1, C)[idx]), oracle.nvfp4_dequantize(want_p, want_s, want_g),
          "unpacked rows")
    del W, p, s, g, y
    torch.cuda.empty_cache()
