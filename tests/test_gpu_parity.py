"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Inputs are seeded and synthetic; the oracle always receives the very bytes
the GPU received (copied back from the device).  Bytes, scales and
dequantized / fake-quantized values must match bit for bit; the grouped
GEMM must satisfy max |y - ref| / max(|ref|, 1e-2 * rms(ref)) <= 1e-2 with
ref the exact (double) sum.
"""
import numpy as np
import pytest
import torch

import full_size_gemm
import nvfp4_quantization_amax_b200 as mxq
import oracle
import synthetic as gen

pytestmark = pytest.mark.gpu

DEV = "cuda"
GEMM_TOL = 1e-2
_NP = {torch.bfloat16: np.uint16, torch.float16: np.uint16, torch.float32: np.uint32}
_INT = {torch.bfloat16: torch.int16, torch.float16: torch.int16, torch.float32: torch.int32}
_NAME = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}


def bits(t):
    """Raw bit patterns of a float tensor as a numpy unsigned array (host)."""
    return t.detach().cpu().contiguous().view(_INT[t.dtype]).numpy().view(_NP[t.dtype])


def u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def assert_bits_equal(got, want, what):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got.reshape(-1) != want.reshape(-1))[0]
    assert bad.size == 0, "%s: %d mismatches, first at %s: got %s want %s" % (
        what, bad.size, bad[:4], got.reshape(-1)[bad[:4]], want.reshape(-1)[bad[:4]])


def gemm_error(y, ref):
    y = np.asarray(y, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return np.max(np.abs(y - ref) / np.maximum(np.abs(ref), 1e-2 * rms))


# ------------------------------------------------------------ MXFP4

def test_mx_small_config_exact():
    x = gen.mx_small(DEV)
    p, s = mxq.mx_quantize(x)
    wp, ws = oracle.mx_quantize(bits(x), "bf16")
    assert_bits_equal(u8(p), wp, "packed")
    assert_bits_equal(u8(s), ws, "scales")
    y = mxq.mx_dequantize(p, s)
    assert_bits_equal(bits(y), oracle.mx_dequantize(wp, ws, "bf16"), "dequant")
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_mx_dequantize_every_byte_and_scale(dtype):
    # row r: every byte value once per 256 bytes, all blocks scaled by byte r
    packed = torch.arange(256, dtype=torch.int32).repeat(256, 1).to(torch.uint8)
    packed = torch.roll(packed, 1, dims=1).contiguous()
    scales = torch.arange(256, dtype=torch.int32).to(torch.uint8)[:, None].repeat(1, 16)
    y = mxq.mx_dequantize(packed.to(DEV), scales.to(DEV), dtype)
    want = oracle.mx_dequantize(packed.numpy(), scales.numpy(), _NAME[dtype])
    assert_bits_equal(bits(y), want, "dequant %s" % dtype)


def f32_edge_values(n, seed):
    """f32 values over the whole exponent range, subnormals included."""
    b = gen.random_bytes(4 * n, seed).view(torch.int32)
    b = b & 0x7FFFFFFF  # drop sign, then draw it again below
    exp = (gen.random_bytes(n, seed + 1).to(torch.int32) % 254) << 23
    man = b & 0x7FFFFF
    sign = (gen.random_bytes(n, seed + 2).to(torch.int32) & 1) << 31
    v = (exp | man | sign).view(torch.float32)
    return v


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_mx_quantize_mixed_blocks_exact(dtype):
    x = gen.mixed_blocks(256, 1024).to(dtype)
    if dtype == torch.float32:
        x.view(-1)[: 256 * 512] = f32_edge_values(256 * 512, 77) * 1e-20
    x = x.to(DEV)
    p, s = mxq.mx_quantize(x)
    wp, ws = oracle.mx_quantize(bits(x), _NAME[dtype])
    assert_bits_equal(u8(s), ws, "scales")
    assert_bits_equal(u8(p), wp, "packed")


def special_blocks():
    """Blocks built to hit every E2M1 decision point exactly, signed zeros,
    saturation, and the extremes of the bf16 range."""
    t8 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    mids = [(a + b) / 2 for a, b in zip(t8[:-1], t8[1:])]
    rows = []
    for e in (-133, -127, -126, -20, 0, 3, 100, 124):  # 8 * 2^124 stays finite
        for sgn in (1.0, -1.0):
            blk = [6.0] + [m * sgn for m in mids] + [(m + 1e-3) * sgn for m in mids] + \
                  [(m - 1e-3) * sgn for m in mids] + [7.0 * sgn, -0.0, 0.0, 5.9 * sgn, 1e-3 * sgn,
                                                       -1e-3, 0.3, 8.0 * sgn, 2.0 ** -20, 4.0]
            rows.append(np.array(blk[:32]) * 2.0 ** e)
    rows.append(np.full(32, -0.0))
    rows.append(np.full(32, 3.3895313892515355e38))  # largest bf16
    x = torch.tensor(np.stack(rows), dtype=torch.float64)
    return x.to(torch.bfloat16)


def test_mx_quantize_decision_points_exact():
    x = special_blocks().to(DEV)
    p, s = mxq.mx_quantize(x)
    wp, ws = oracle.mx_quantize(bits(x), "bf16")
    assert_bits_equal(u8(s), ws, "scales")
    assert_bits_equal(u8(p), wp, "packed")


def test_mx_expert_weights_full_size_sampled():
    # full-size expert weight pack [64, 2048, 7168] and unpack, as timed
    W = gen.expert_weights(device=DEV)
    p, s = mxq.mx_quantize(W)
    y = mxq.mx_dequantize(p, s)
    rows = torch.randperm(64 * 2048, generator=torch.Generator().manual_seed(3))[:96]
    rows = torch.cat([rows, torch.tensor([0, 64 * 2048 - 1])])
    Wr = W.view(-1, 7168)[rows.to(DEV)]
    wp, ws = oracle.mx_quantize(bits(Wr), "bf16")
    assert_bits_equal(u8(p.view(-1, 3584)[rows.to(DEV)]), wp, "packed rows")
    assert_bits_equal(u8(s.view(-1, 224)[rows.to(DEV)]), ws, "scale rows")
    assert_bits_equal(bits(y.view(-1, 7168)[rows.to(DEV)]), oracle.mx_dequantize(wp, ws, "bf16"),
                      "dequant rows")
    # at any size: unpack(pack(unpack(q))) == unpack(q)
    p2, s2 = mxq.mx_quantize(y)
    y2 = mxq.mx_dequantize(p2, s2)
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    assert int(s.max()) < 255
    del W, p, s, y, p2, s2, y2
    torch.cuda.empty_cache()


@pytest.mark.parametrize("R", [1024, 4096])
def test_mx_mixed_blocks_rows(R):
    x = gen.mixed_blocks(R, 7168, device=DEV)
    p, s = mxq.mx_quantize(x)
    wp, ws = oracle.mx_quantize(bits(x), "bf16")
    assert_bits_equal(u8(s), ws, "scales")
    assert_bits_equal(u8(p), wp, "packed")
    y = mxq.mx_dequantize(p, s)
    assert_bits_equal(bits(y), oracle.mx_dequantize(wp, ws, "bf16"), "dequant")


def test_mx_ragged_tail_items():
    # rows*K/8 not a multiple of the warp width: the last warp is partial
    x = gen.mixed_blocks(3, 96, device=DEV)
    p, s = mxq.mx_quantize(x)
    wp, ws = oracle.mx_quantize(bits(x), "bf16")
    assert_bits_equal(u8(p), wp, "packed")
    assert_bits_equal(u8(s), ws, "scales")


# ----------------------------------------------------- quantize_cache

@pytest.mark.parametrize("fmt,B", [("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_cache_kv_full_size_exact(fmt, B):
    x = gen.kv_cache(device=DEV)
    y = mxq.quantize_cache(x, fmt, B)
    assert y.shape == x.shape and y.dtype == x.dtype and y.data_ptr() != x.data_ptr()
    assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), fmt, B), "%s B=%d" % (fmt, B))


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("B", [8, 16, 32, 64, 128, 256])
def test_cache_fast_block_sizes(fmt, B):
    x = torch.cat([gen.kv_cache((1, 64, 512)).view(64, 512), gen.mixed_blocks(64, 512)]).to(DEV)
    y = mxq.quantize_cache(x, fmt, B)
    assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), fmt, B), "%s B=%d" % (fmt, B))


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_cache_other_dtypes(fmt, dtype):
    x = torch.cat([gen.kv_cache((1, 64, 512)).view(64, 512), gen.mixed_blocks(64, 512)]).to(dtype)
    if dtype == torch.float32:
        x.view(-1)[:8192] = f32_edge_values(8192, 5) * 1e-30
    x = x.to(DEV)
    for B in (16, 32, 128):
        y = mxq.quantize_cache(x, fmt, B)
        assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), fmt, B, _NAME[dtype]),
                          "%s %s B=%d" % (fmt, dtype, B))


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("C,B", [(40, 16), (520, 32), (100, 7), (33, 1), (7, 3), (130, 128)])
def test_cache_general_shapes(fmt, C, B):
    x = gen.kv_cache((1, 37, C)).view(37, C).to(DEV)
    y = mxq.quantize_cache(x, fmt, B)
    assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), fmt, B), "%s C=%d B=%d" % (fmt, C, B))


def test_cache_unaligned_input_takes_general_path():
    base = gen.kv_cache((1, 17, 257)).view(-1).to(DEV)
    x = torch.as_strided(base, (16, 256), (256, 1), 1)  # offset by one element
    y = mxq.quantize_cache(x, "nvfp4", 16)
    assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), "nvfp4", 16), "unaligned")


@pytest.mark.parametrize("fmt,B", [("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_cache_mixed_rows_exact(fmt, B):
    x = gen.mixed_blocks(1024, 7168, device=DEV)
    y = mxq.quantize_cache(x, fmt, B)
    assert_bits_equal(bits(y), oracle.quantize_cache(bits(x), fmt, B), "%s mixed" % fmt)


def test_cache_idempotent_on_gpu():
    x = gen.kv_cache(device=DEV)
    for fmt, B in (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)):
        y = mxq.quantize_cache(x, fmt, B)
        assert torch.equal(mxq.quantize_cache(y, fmt, B).view(torch.int16), y.view(torch.int16))


# ------------------------------------------------------- grouped GEMM

def moe_case(counts, N, K, seed=21, scale_lo=116, scale_hi=124):
    E = len(counts)
    offs = torch.tensor(np.cumsum(counts), dtype=torch.int32)
    T = int(offs[-1])
    packed, scales = gen.random_packed(E, N, K, scale_lo, scale_hi, workload=seed)
    x = gen.normal_bf16(gen.seed_for(seed, 3), (T, K))
    g = gen.normal_bf16(gen.seed_for(seed, 4), (T, N))
    return x, g, packed, scales, offs


def check_gemm(counts, N, K, transpose_w, rows=None, seed=21, scale_lo=116, scale_hi=124):
    x, g, packed, scales, offs = moe_case(counts, N, K, seed, scale_lo, scale_hi)
    a = g if transpose_w else x
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a.to(DEV), packed.to(DEV), scales.to(DEV), offs.to(DEV),
                             transpose_w=transpose_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.grouped_mm(bits(a), packed.numpy(), scales.numpy(), offs.numpy(),
                            transpose_w=transpose_w, rows=rows)
    yv = oracle.decode(bits(y), "bf16")
    if rows is not None:
        yv = yv[np.asarray(rows)]
    err = gemm_error(yv, ref)
    assert err <= GEMM_TOL, err
    return err


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_ragged_experts(transpose_w):
    # several tiles, ragged tails, an empty expert and a one-row expert
    check_gemm([300, 0, 1, 257, 130, 512], N=256, K=512, transpose_w=transpose_w)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_scales_above_the_benchmark_range(transpose_w):
    # scale bytes 136..150: larger weights than the benchmark's (the whole
    # 0..252 range is covered per expert in test_gpu_gemm_edges.py)
    check_gemm([129, 64, 300], N=256, K=256, transpose_w=transpose_w, scale_lo=136,
               scale_hi=150)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_many_small_experts(transpose_w):
    # 40 experts of 0..40 rows: every tail width, many tiles per CTA
    counts = [(7 * i) % 41 for i in range(40)]
    check_gemm(counts, N=128, K=128, transpose_w=transpose_w)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_general_shapes(transpose_w):
    check_gemm([5, 0, 17, 40], N=100, K=96, transpose_w=transpose_w)


def test_grouped_mm_bad_offs_reports_status():
    x, g, packed, scales, _ = moe_case([8, 8], 128, 64)
    y = torch.full((16, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    for offs in ([9, 8], [8, 15], [-1, 16]):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        mxq.mxfp4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV),
                             torch.tensor(offs, dtype=torch.int32, device=DEV), out=y,
                             status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -6
        assert bool((y == 7.0).all())


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_full_size_sampled(transpose_w):
    T, E, N, K = 32768, 32, 2048, 7168
    counts = gen.expert_counts(T, E).numpy()
    offs = np.cumsum(counts)
    starts = np.concatenate([[0], offs[:-1]])
    rng = np.random.default_rng(8)
    rows = []
    for lo, hi in zip(starts, offs):
        if hi > lo:
            rows += [lo, hi - 1] + list(rng.integers(lo, hi, 2))
    rows = np.unique(np.array(rows, np.int64))
    hp, hs, packed, scales = full_size_gemm.packed_weights(DEV)  # packed by the oracle
    a = gen.normal_bf16(gen.seed_for(5, 4 if transpose_w else 3), (T, N if transpose_w else K),
                        device=DEV)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a, packed, scales, offs_d, transpose_w=transpose_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.grouped_mm(bits(a), hp, hs, offs.astype(np.int32),
                            transpose_w=transpose_w, rows=rows)
    yv = oracle.decode(bits(y[torch.tensor(rows, device=DEV)]), "bf16")
    assert gemm_error(yv, ref) <= GEMM_TOL


def test_grouped_mm_wait_timeout_reports_status():
    # A zero wait limit makes the first pipeline wait that is not already
    # satisfied give up: the kernel must drain, free TMEM and report
    # MXQ_ERR_TIMEOUT, and the context must stay usable.
    x, g, packed, scales, offs = moe_case([700, 300, 50], N=128, K=512)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    prev = mxq.set_wait_limit_ns(0)
    try:
        mxq.mxfp4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV), offs.to(DEV),
                             status=status)
        torch.cuda.synchronize()
    finally:
        mxq.set_wait_limit_ns(prev)
    assert int(status.item()) == -7
    check_gemm([700, 300, 50], N=128, K=512, transpose_w=False)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_wait_timeout_pair_shape(transpose_w):
    # The same on the CTA-pair kernel (output width a multiple of 256): after
    # the abort both CTAs' activation loads are settled and drained before
    # either CTA exits, and the context stays usable.
    counts = [700, 300, 50]
    x, g, packed, scales, offs = moe_case(counts, N=256, K=512)
    a = g if transpose_w else x
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    prev = mxq.set_wait_limit_ns(0)
    try:
        mxq.mxfp4_grouped_mm(a.to(DEV), packed.to(DEV), scales.to(DEV), offs.to(DEV),
                             transpose_w=transpose_w, status=status)
        torch.cuda.synchronize()
    finally:
        mxq.set_wait_limit_ns(prev)
    assert int(status.item()) == -7
    check_gemm(counts, N=256, K=512, transpose_w=transpose_w)


# ------------------------------------------------------- NVFP4 two-level

def nv_inputs(dtype):
    x = torch.cat([gen.kv_cache((1, 64, 512)).view(64, 512), gen.mixed_blocks(64, 512),
                   gen.normal_bf16(41, (64, 512))]).to(dtype)
    if dtype == torch.float32:
        x.view(-1)[:4096] = f32_edge_values(4096, 9) * 1e-25
    return x


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_nvfp4_quantize_exact(dtype):
    x = nv_inputs(dtype).to(DEV)
    p, s, g = mxq.nvfp4_quantize(x)
    wp, ws, wg = oracle.nvfp4_quantize(bits(x), _NAME[dtype])
    assert float(g.item()) == wg
    assert_bits_equal(u8(s), ws, "block scales")
    assert_bits_equal(u8(p), wp, "packed")


def test_nvfp4_expert_weights_exact():
    x = gen.expert_weights(4, 2048, 7168, device=DEV)
    p, s, g = mxq.nvfp4_quantize(x)
    wp, ws, wg = oracle.nvfp4_quantize(bits(x))
    assert float(g.item()) == wg
    assert_bits_equal(u8(s), ws, "block scales")
    assert_bits_equal(u8(p), wp, "packed")
    assert int(s.max()) == 0x7E  # the top block is scaled by exactly 448


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_nvfp4_dequantize_exact(dtype):
    wp, ws, wg = oracle.nvfp4_quantize(bits(nv_inputs(torch.bfloat16)))
    y = mxq.nvfp4_dequantize(torch.from_numpy(wp).to(DEV), torch.from_numpy(ws).to(DEV),
                             torch.tensor([wg], dtype=torch.float32, device=DEV), dtype)
    assert_bits_equal(bits(y), oracle.nvfp4_dequantize(wp, ws, wg, _NAME[dtype]), "dequant")


@pytest.mark.parametrize("rule", ["max", "mse"])
def test_nvfp4_blocks_far_below_the_tensor_max(rule):
    # block-scale quotients below 2^-9 clamp to the smallest E4M3 scale
    # (byte 0x01) under the max rule; values of a few 2^-9 g still get codes
    grid = 2.0**-9 / 2688.0
    x = torch.zeros(4, 64)
    x[0, 0] = 1.0
    x[0, 1:64] = gen.normal_bf16(43, (63,)).float() * 0.25
    for r in range(1, 4):
        x[r] = torch.tensor([(0.3 + 0.09 * i) * grid * r * (-1) ** i for i in range(64)])
    x = x.to(torch.bfloat16).to(DEV)
    p, s, g = mxq.nvfp4_quantize(x, rule=rule)
    fn = oracle.nvfp4_quantize if rule == "max" else oracle.nvfp4_quantize_mse
    wp, ws, wg = fn(bits(x))
    assert float(g.item()) == wg
    assert_bits_equal(u8(s), ws, "block scales")
    assert_bits_equal(u8(p), wp, "packed")
    if rule == "max":
        assert int(u8(s)[1].min()) == 0x01


@pytest.mark.parametrize("rule", ["max", "mse"])
def test_nvfp4_sign_follows_x_where_the_quotient_underflows(rule):
    x = torch.zeros(2, 32)
    x[0, 0] = 1e30
    x[0, 1:8] = torch.tensor([-1e-20, -1e-20, 1e-20, -3e-25, 2.5e28, -7e27, -1e-30])
    x[1] = gen.normal_bf16(44, (32,)).float() * 1e-19
    x = x.to(torch.bfloat16).to(DEV)
    p, s, g = mxq.nvfp4_quantize(x, rule=rule)
    fn = oracle.nvfp4_quantize if rule == "max" else oracle.nvfp4_quantize_mse
    wp, ws, wg = fn(bits(x))
    assert float(g.item()) == wg
    assert_bits_equal(u8(s), ws, "block scales")
    assert_bits_equal(u8(p), wp, "packed")
    assert (int(u8(p)[0, 0]) >> 4) == 8 and (int(u8(p)[0, 1]) & 15) == 8


def test_nvfp4_zero_and_ragged():
    z = torch.zeros(3, 48, dtype=torch.bfloat16, device=DEV)
    p, s, g = mxq.nvfp4_quantize(z)
    assert float(g.item()) == 0.0 and int(p.max()) == 0 and bool((s == 0x38).all())
    x = gen.normal_bf16(77, (5, 48), device=DEV)  # 30 items: a partial warp
    p, s, g = mxq.nvfp4_quantize(x)
    wp, ws, wg = oracle.nvfp4_quantize(bits(x))
    assert float(g.item()) == wg
    assert_bits_equal(u8(p), wp, "packed")
    assert_bits_equal(u8(s), ws, "scales")


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_small_remainders(transpose_w):
    # experts just above a multiple of the 256-row tile (remainders of 1,
    # 31, 32, 33, 63, 64 and 65 rows), one-row and empty experts: every
    # ragged tail the CTA-pair tiling meets
    counts = [257, 287, 288, 289, 319, 320, 321, 576, 600, 64, 1, 0, 512]
    check_gemm(counts, 256, 512, transpose_w)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_scale_rows_not_16_byte_multiples(transpose_w):
    # K = 768: 24 scale bytes per weight row, so the weight tiles are staged
    # by TMA but their scale bytes are read from global memory
    check_gemm([130, 300, 90], N=256, K=768, transpose_w=transpose_w)


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_more_experts_than_the_offs_cache(transpose_w):
    # 300 experts (more than the shared-memory copy of offs holds): the tile
    # walks read offs from global memory
    counts = [int(c) for c in np.random.RandomState(3).randint(0, 9, size=300)]
    check_gemm(counts, N=256, K=256, transpose_w=transpose_w)
