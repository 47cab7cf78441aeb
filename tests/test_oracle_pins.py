"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute from its
own tables: values the pages print (tests/golden/, each with its citation),
brute force over every bf16 bit pattern, library casts (torch, numpy), closed
forms and invariants of the method.  A plausible slip in the oracle - a wrong
midpoint, a tie broken the wrong way, a swapped nibble, an off-by-one in a
scale exponent, a dropped sign, a transposed GEMM operand - fails at least
one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic as gen
from conftest import read_golden

# The eight E2M1 magnitudes as the page prints them (codes 0..7).
PAGE_TABLE = {int(i): float(v) for i, v in read_golden("e2m1_table.txt")}
T8 = np.array([PAGE_TABLE[i] for i in range(8)])
MIDPOINTS = [float(v) for v in read_golden("e2m1_midpoints.txt")[0]]


def all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f32 = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(f32)
    with np.errstate(invalid="ignore"):  # signalling-NaN patterns; dropped below
        vals = f32.astype(np.float64)
    return bits[keep], vals[keep]


def bruteforce_e2m1_mag(a):
    """Index of the nearest of T8 to a >= 0; on a tie the even index."""
    d = np.abs(a[:, None] - T8[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    idx = np.where(cand, np.arange(8)[None, :], 99)
    even = np.where(cand & (np.arange(8)[None, :] % 2 == 0), np.arange(8)[None, :], 99)
    return np.where(even.min(axis=1) < 99, even.min(axis=1), idx.min(axis=1))


def e4m3_candidates():
    """(value, code) of the 127 non-negative finite E4M3 numbers, built from
    the format definition (bias 7, 3 mantissa bits, S.1111.111 is NaN)."""
    out = [(m * 2.0 ** -9, m) for m in range(8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            out.append(((8 + m) * 2.0 ** (e - 10), (e << 3) | m))
    return np.array([v for v, _ in out]), np.array([c for _, c in out])


def bruteforce_e4m3(vals):
    cv, cc = e4m3_candidates()
    a = np.abs(vals)
    d = np.abs(a[:, None] - cv[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = cand & (cc[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
    r = cv[pick]
    r = np.where(a > 448.0, 448.0, r)
    return np.copysign(r, vals)


# ---------------------------------------------------------------- E2M1 table

def test_table_matches_page():
    for i, v in PAGE_TABLE.items():
        assert oracle.e2m1_value(i) == v, i
    # index 8 prints as 0.0: a positive zero
    assert math.copysign(1.0, oracle.e2m1_value(8)) == 1.0


def test_table_sign_half():
    # codes 8..15 carry the sign bit of 0..7 (codes 13..15 are not printed)
    for c in range(1, 8):
        assert oracle.e2m1_value(c + 8) == -T8[c]


def test_midpoints_are_means_of_neighbours():
    assert len(MIDPOINTS) == 7
    for i, m in enumerate(MIDPOINTS):
        assert m == (T8[i] + T8[i + 1]) / 2


@pytest.mark.parametrize("row", read_golden("e2m1_ties.txt"))
def test_tie_rule_from_page(row):
    tie, want = float(row[0]), float(row[1])
    assert oracle.e2m1_value(oracle.e2m1_code(tie)) == want
    assert oracle.e2m1_value(oracle.e2m1_code(-tie)) == -want


def test_e2m1_code_bruteforce_every_bf16():
    _, vals = all_finite_bf16()
    # distances are exact in double only while |v| < 2^40; beyond, the
    # nearest magnitude is 6 (code 7) by definition
    big = np.abs(vals) >= 2.0**40
    mag = np.where(big, 7, bruteforce_e2m1_mag(np.where(big, 0.0, np.abs(vals))))
    want = mag | np.where(vals < 0, 8, 0)
    got = np.array([oracle.e2m1_code(v) for v in vals])
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e2m1_sign_reading():
    # -0.0 carries no sign bit; a tiny negative keeps it (nibble 8)
    assert oracle.e2m1_code(-0.0) == 0
    assert oracle.e2m1_code(-1e-30) == 8
    assert oracle.e2m1_code(-7.0) == 15


# ------------------------------------------------------- binary formats

def test_e4m3_rounding_bruteforce_every_bf16():
    _, vals = all_finite_bf16()
    vals = vals[np.abs(vals) < 1e6]
    want = bruteforce_e4m3(vals)
    got = np.array([oracle.round_e4m3(v) for v in vals])
    assert np.array_equal(np.signbit(got), np.signbit(want))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_rounding_matches_torch_cast():
    _, vals = all_finite_bf16()
    vals = vals[np.abs(vals) <= 448.0]
    t = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64)
    got = np.array([oracle.round_e4m3(v) for v in vals])
    assert np.array_equal(got, t.numpy())


def test_e4m3_encode_decode_all_bytes():
    cv, cc = e4m3_candidates()
    byval = dict(zip(cc.tolist(), cv.tolist()))
    for b in range(256):
        mag = b & 0x7F
        if mag == 0x7F:
            assert math.isnan(oracle.decode_e4m3(b))
            continue
        v = oracle.decode_e4m3(b)
        assert abs(v) == byval[mag]
        assert math.copysign(1.0, v) == (-1.0 if b & 0x80 else 1.0)
        assert oracle.encode_e4m3(v) == b


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32)
    edge = np.array([0x00000001, 0x00008000, 0x00007FFF, 0x00018000, 0x007FFFFF, 0x00800000,
                     0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0x3F808000, 0x3F818000, 0x80000001,
                     0xFF7F8000, 0x00000000, 0x80000000], np.uint32)
    bits = np.concatenate([bits, edge])
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_to(f.astype(np.float64), "bf16")
    assert np.array_equal(got, want)


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.standard_normal(100000) * 10.0 ** rng.uniform(-9, 5, 100000),
        np.array([65504.0, 65519.99, 65520.0, 2.0**-24, 2.0**-25, 3 * 2.0**-26, 2.0**-14,
                  -0.0, 0.0, 1 + 2.0**-11, 1 + 3 * 2.0**-11])])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.round_to(v, "f16"), want)


def _same_values(got, want):
    nan = np.isnan(want)
    return (np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], want[~nan])
            and np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan])))


def test_every_f16_and_bf16_pattern_decodes_like_the_libraries():
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    assert _same_values(oracle.decode(allb, "f16"), allb.view(np.float16).astype(np.float64))
    want = torch.from_numpy(allb.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert _same_values(oracle.decode(allb, "bf16"), want)


def test_f32_patterns_decode_like_numpy():
    rng = np.random.default_rng(5)
    u = np.concatenate([rng.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32),
                        np.array([0, 0x80000000, 1, 0x807FFFFF, 0x7F7FFFFF, 0x7F800000, 0xFF800000,
                                  0x00800000], dtype=np.uint32)])
    with np.errstate(invalid="ignore"):  # numpy flags signalling NaNs as it widens them
        want = u.view(np.float32).astype(np.float64)
    assert _same_values(oracle.decode(u, "f32"), want)


def test_f32_rounding_matches_numpy():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(100000) * 10.0 ** rng.uniform(-45, 38, 100000)
    v = np.concatenate([v, [2.0**-149, 2.0**-150, 3 * 2.0**-151, 3.4028235677973366e38]])
    with np.errstate(over="ignore"):
        want = v.astype(np.float32).view(np.uint32)
    assert np.array_equal(oracle.round_to(v, "f32"), want)


# ------------------------------------------------------- MXFP4 pack / unpack

def full_table():
    return np.array([PAGE_TABLE.get(c, -T8[c - 8] if c >= 8 else None) for c in range(16)])


def test_every_byte_decodes_low_nibble_first():
    tab = full_table()
    packed = np.arange(256, dtype=np.uint8).reshape(1, 256)
    scales = np.full((1, 16), 127, np.uint8)
    out = oracle.decode(oracle.mx_dequantize(packed, scales, "f32"), "f32")[0]
    b = np.arange(256)
    assert np.array_equal(out[0::2], tab[b & 15])
    assert np.array_equal(out[1::2], tab[b >> 4])


def test_scale_byte_is_power_of_two():
    for s in range(256):
        packed = np.full((1, 16), 0x22, np.uint8)  # two codes 2 (= 1.0)
        scales = np.array([[s]], np.uint8)
        out = oracle.decode(oracle.mx_dequantize(packed, scales, "f32"), "f32")[0]
        if s == 255:
            assert np.isnan(out).all()
        else:
            assert (out == math.ldexp(1.0, s - 127)).all(), s


def test_every_byte_round_trips():
    # byte b beside a 0x77 byte (two 6.0s) so the block max is 6 and the
    # derived scale is 2^0 again
    for b in range(256):
        packed = np.zeros((1, 16), np.uint8)
        packed[0, 0] = b
        packed[0, 1] = 0x77
        scales = np.array([[127]], np.uint8)
        x = oracle.mx_dequantize(packed, scales, "bf16")
        p2, s2 = oracle.mx_quantize(x, "bf16")
        assert s2[0, 0] == 127
        lo, hi = b & 15, b >> 4
        lo, hi = (0 if lo == 8 else lo), (0 if hi == 8 else hi)  # +0.0 re-encodes as nibble 0
        assert p2[0, 0] == lo | (hi << 4), b
        assert p2[0, 1] == 0x77


def test_dequant_quant_dequant_is_identity():
    # the value-exact round trip quantize_mxfp4 promises for exactly
    # representable inputs, over every scale byte that stays finite in bf16
    rng = np.random.default_rng(4)
    rows = 253
    packed = rng.integers(0, 256, (rows, 64), dtype=np.uint8)
    scales = np.repeat(np.arange(rows, dtype=np.uint8)[:, None], 4, axis=1)
    x = oracle.mx_dequantize(packed, scales, "bf16")
    p2, s2 = oracle.mx_quantize(x, "bf16")
    x2 = oracle.mx_dequantize(p2, s2, "bf16")
    assert np.array_equal(oracle.decode(x2, "bf16"), oracle.decode(x, "bf16"))


def test_scale_rule_floor_log2_minus_2():
    x = gen.mixed_blocks(64, 256).view(torch.int16).numpy().view(np.uint16)
    vals = oracle.decode(x, "bf16").reshape(-1, 32)
    _, s = oracle.mx_quantize(x, "bf16")
    s = s.reshape(-1).astype(int)
    for blk, byte in zip(vals, s):
        amax = np.abs(blk).max()
        if amax == 0:
            assert byte == 0
            continue
        e = byte - 127
        fl = math.frexp(amax)[1] - 1  # floor(log2 amax)
        assert e == max(fl - 2, -127)
        if e > -127:
            assert 2.0 ** (e + 2) <= amax < 2.0 ** (e + 3)


def test_forced_rows_closed_form():
    x = gen.mx_small().view(torch.int16).numpy().view(np.uint16)
    p, s = oracle.mx_quantize(x, "bf16")
    # row 0 all zero: scale byte 0, codes 0
    assert (p[0] == 0).all() and (s[0] == 0).all()
    # row 1 all 1.75: floor(log2 1.75) - 2 = -2 -> byte 125; 1.75/2^-2 = 7 saturates to 6 (code 7)
    assert (s[1] == 125).all() and (p[1] == 0x77).all()
    # row 2: block max exactly 2 -> e = -1 (byte 126); the +-2 element is 4.0 = code 6 (+8 if negative)
    assert (s[2] == 126).all()
    xv = oracle.decode(x[2], "bf16")
    codes = np.stack([p[2] & 15, p[2] >> 4], axis=1).reshape(-1)
    two = np.abs(xv) == 2.0
    assert two.sum() == 8
    assert np.array_equal(codes[two], np.where(xv[two] < 0, 14, 6))
    # row 3 all 2^-3: e = -5 (byte 122); 2^-3 / 2^-5 = 4 -> code 6
    assert (s[3] == 122).all() and (p[3] == 0x66).all()


def test_mx_quantize_bruteforce_tiny():
    rng = np.random.default_rng(5)
    tab = full_table()
    for trial in range(200):
        v = rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 3)
        bits = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        xv = oracle.decode(bits, "bf16")
        p, s = oracle.mx_quantize(bits.reshape(1, 32), "bf16")
        amax = np.abs(xv).max()
        e = max(math.frexp(amax)[1] - 1 - 2, -127)
        assert s[0, 0] == e + 127
        scaled = xv / 2.0 ** e
        codes = np.stack([p[0] & 15, p[0] >> 4], axis=1).reshape(-1)
        for j in range(32):
            d = np.abs(scaled[j] - tab)
            cands = np.nonzero(d == d.min())[0]
            # among equally near codes: the sign must follow v<0, ties go to the even magnitude
            cands = [c for c in cands if (c >= 8) == (scaled[j] < 0) or tab[c] == 0]
            mags = sorted({c & 7 for c in cands}, key=lambda m: (m % 2, m))
            want = mags[0] | (8 if scaled[j] < 0 else 0)
            assert codes[j] == want, (trial, j, scaled[j])


def test_effective_bits_ratio(facts):
    x = gen.normal_bf16(9, (4, 7168)).view(torch.int16).numpy().view(np.uint16)
    p, s = oracle.mx_quantize(x, "bf16")
    assert s.nbytes * 16 == p.nbytes  # MXFP4: 8 scale bits per 32 values of 4 bits
    assert facts["r1_fp4_scale_bytes"] * 8 == facts["r1_fp4_packed_bytes"]
    assert facts["expert_cols"] / 2 == facts["expert_packed_cols"]
    assert facts["expert_cols"] / facts["nvfp4_block_size"] == facts["expert_nvfp4_scale_cols"]
    assert 4 + 8 / facts["nvfp4_block_size"] == facts["nvfp4_effective_bits"]


# ----------------------------------------------------- quantize_cache

QMAX = {"fp8": 448.0, "mxfp4": 6.0, "nvfp4": 6.0}
CLAMP = {"fp8": (-126, 127), "mxfp4": (-126, 127), "nvfp4": (-9, 8)}


def independent_scale_exp(amax, fmt):
    lo, hi = CLAMP[fmt]
    if amax == 0:
        return lo
    k = -300
    while QMAX[fmt] * 2.0 ** k < amax:  # exact: powers of two times 448 or 6
        k += 1
    return min(max(k, lo), hi)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
def test_cache_scale_is_power_of_two_ceiling(fmt):
    _, vals = all_finite_bf16()
    amaxes = np.unique(np.abs(vals))
    for a in amaxes[::7]:
        assert oracle.cache_scale_exp(a, fmt) == independent_scale_exp(a, fmt), a
    q = QMAX[fmt]
    assert oracle.cache_scale_exp(q, fmt) == 0
    assert oracle.cache_scale_exp(np.nextafter(q, 10 * q), fmt) == 1
    assert oracle.cache_scale_exp(q / 2, fmt) == -1


def cache_bruteforce(xv, fmt, B):
    """Fake quantization by nearest-grid search: for each group the scale is
    the least power of two with 2^k*qmax >= amax; each value goes to the
    nearest grid point (ties: even code), zero magnitudes are +0 for the fp4
    formats and keep their sign for fp8; then nearest-even to bf16."""
    out = np.empty_like(xv)
    cv, cc = e4m3_candidates()
    for r in range(xv.shape[0]):
        for c0 in range(0, xv.shape[1], B):
            blk = xv[r, c0:c0 + B]
            k = independent_scale_exp(np.abs(blk).max(), fmt)
            v = blk / 2.0 ** k
            if fmt == "fp8":
                q = bruteforce_e4m3(v)
            else:
                mag = bruteforce_e2m1_mag(np.abs(v))
                q = np.where(mag == 0, 0.0, np.copysign(T8[mag], v))
            out[r, c0:c0 + B] = q * 2.0 ** k
    f32 = out.astype(np.float32)  # exact: at most 4 significant bits, >= 2^-135
    assert np.array_equal(f32.astype(np.float64), out)
    return torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("fmt,B", [("fp8", 128), ("fp8", 32), ("mxfp4", 32), ("nvfp4", 16),
                                   ("nvfp4", 7)])
def test_cache_matches_nearest_grid_bruteforce(fmt, B):
    x = torch.cat([gen.kv_cache((1, 6, 256)).view(6, 256), gen.mixed_blocks(6, 256)])
    bits = x.view(torch.int16).numpy().view(np.uint16)
    got = oracle.quantize_cache(bits, fmt, B)
    want = cache_bruteforce(oracle.decode(bits, "bf16"), fmt, B)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt,B", [("fp8", 32), ("mxfp4", 32), ("nvfp4", 16)])
def test_cache_tail_group_is_zero_padded(fmt, B):
    # a final partial group behaves as if zero-padded to a full group
    x = gen.kv_cache((1, 5, 48)).view(5, 48).clone()
    x[:, 40:] = 0.0
    bits = x.view(torch.int16).numpy().view(np.uint16)
    full = oracle.quantize_cache(bits, fmt, B)
    part = oracle.quantize_cache(np.ascontiguousarray(bits[:, :40]), fmt, B)
    assert np.array_equal(part, full[:, :40])


@pytest.mark.parametrize("fmt,B", [("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_cache_is_idempotent(fmt, B):
    x = torch.cat([gen.kv_cache((1, 16, 512)).view(16, 512), gen.mixed_blocks(16, 512)])
    bits = x.view(torch.int16).numpy().view(np.uint16)
    once = oracle.quantize_cache(bits, fmt, B)
    twice = oracle.quantize_cache(once, fmt, B)
    assert np.array_equal(once, twice)


def test_cache_fp8_matches_torch_cast():
    x = gen.kv_cache((1, 32, 256)).view(32, 256)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xv = oracle.decode(bits, "bf16")
    want = np.empty_like(xv)
    for r in range(32):
        for c0 in range(0, 256, 32):
            blk = xv[r, c0:c0 + 32]
            k = independent_scale_exp(np.abs(blk).max(), "fp8")
            q = torch.from_numpy((blk / 2.0 ** k).astype(np.float32)).to(torch.float8_e4m3fn)
            want[r, c0:c0 + 32] = q.to(torch.float64).numpy() * 2.0 ** k
    w = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = oracle.quantize_cache(bits, "fp8", 32)
    assert np.array_equal(got, w.view(np.uint16))


def test_cache_clamps():
    # nvfp4: a block of ~1e-40 values takes the 2^-9 floor and rounds to +0
    tiny = torch.full((1, 16), 1e-40, dtype=torch.bfloat16).view(torch.int16).numpy()
    out = oracle.quantize_cache(tiny.view(np.uint16), "nvfp4", 16)
    assert (out == 0).all()
    # nvfp4: a block with max 1e4 takes the 2^8 ceiling and saturates at 6*256
    big = torch.tensor([[1e4] + [1.0] * 15], dtype=torch.bfloat16).view(torch.int16).numpy()
    out = oracle.decode(oracle.quantize_cache(big.view(np.uint16), "nvfp4", 16), "bf16")
    assert out[0, 0] == 1536.0
    # fp8: tiny values keep the sign of zero
    neg = torch.tensor([[-1e-30, 1.0] + [0.0] * 30], dtype=torch.bfloat16).view(torch.int16)
    out = oracle.decode(oracle.quantize_cache(neg.numpy().view(np.uint16), "fp8", 32), "bf16")
    assert out[0, 0] == 0.0 and math.copysign(1.0, out[0, 0]) == -1.0
    # mxfp4: tiny negatives become +0
    out = oracle.decode(oracle.quantize_cache(neg.numpy().view(np.uint16), "mxfp4", 32), "bf16")
    assert out[0, 0] == 0.0 and math.copysign(1.0, out[0, 0]) == 1.0


# ----------------------------------------------------- grouped GEMM

def small_moe(T=7, counts=(3, 0, 4), N=5, K=64, seed=11):
    E = len(counts)
    offs = np.cumsum(counts).astype(np.int32)
    assert offs[-1] == T
    packed, scales = gen.random_packed(E, N, K, 118, 130, workload=seed)
    a = gen.normal_bf16(seed, (T, K)).view(torch.int16).numpy().view(np.uint16)
    return a, packed.numpy(), scales.numpy(), offs


def dense_weights(packed, scales):
    E = packed.shape[0]
    return np.stack([oracle.decode(oracle.mx_dequantize(packed[e], scales[e], "f32"), "f32")
                     for e in range(E)])


def test_grouped_mm_forward_matches_numpy():
    a, packed, scales, offs = small_moe()
    W = dense_weights(packed, scales)
    av = oracle.decode(a, "bf16")
    got = oracle.grouped_mm(a, packed, scales, offs)
    lo = 0
    for e, hi in enumerate(offs):
        want = av[lo:hi] @ W[e].T
        np.testing.assert_allclose(got[lo:hi], want, rtol=1e-12, atol=1e-300)
        lo = hi


def test_grouped_mm_dgrad_matches_numpy():
    a, packed, scales, offs = small_moe()
    N = packed.shape[1]
    g = gen.normal_bf16(12, (7, N)).view(torch.int16).numpy().view(np.uint16)
    W = dense_weights(packed, scales)
    gv = oracle.decode(g, "bf16")
    got = oracle.grouped_mm(g, packed, scales, offs, transpose_w=True)
    lo = 0
    for e, hi in enumerate(offs):
        np.testing.assert_allclose(got[lo:hi], gv[lo:hi] @ W[e], rtol=1e-12, atol=1e-300)
        lo = hi


def test_grouped_mm_one_hot_rows_pick_weights():
    _, packed, scales, offs = small_moe()
    W = dense_weights(packed, scales)
    K = packed.shape[2] * 2
    T = int(offs[-1])
    a = np.zeros((T, K), np.float32)
    ks = [(3 * t + 1) % K for t in range(T)]
    for t, k in enumerate(ks):
        a[t, k] = 1.0
    bits = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.grouped_mm(bits, packed, scales, offs)
    expert = np.searchsorted(offs, np.arange(T), side="right")
    for t in range(T):
        assert np.array_equal(got[t], W[expert[t], :, ks[t]])


def test_grouped_mm_rejects_bad_offs():
    a, packed, scales, _ = small_moe()
    with pytest.raises(ValueError):
        oracle.grouped_mm(a, packed, scales, np.array([3, 2, 7], np.int32))
    with pytest.raises(ValueError):
        oracle.grouped_mm(a, packed, scales, np.array([3, 3, 6], np.int32))
    assert oracle.check_offs(np.array([0, 0, 7], np.int32), 7)


# ----------------------------------------------------- NVFP4 two-level

def e2m1_bruteforce_code(v):
    """Nearest E2M1 code of a finite value (ties to the even magnitude),
    sign bit iff v < 0 (a -0.0 quotient of a negative input keeps it below)."""
    mag = int(bruteforce_e2m1_mag(np.array([abs(v)]))[0]) if abs(v) < 2.0**40 else 7
    return mag


def nvfp4_reference(xv):
    """NVFP4 two-level quantization computed with numpy binary32 arithmetic
    and torch's E4M3 cast (independent of the oracle's own routines)."""
    f32 = np.float32
    amax = f32(np.abs(xv).max())
    rows, K = xv.shape
    packed = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    if amax == 0:
        scales[:] = torch.tensor([1.0]).to(torch.float8_e4m3fn).view(torch.uint8).item()
        return packed, scales, 0.0
    g = f32(amax) / f32(2688.0)
    t = f32(6.0) * g
    for r in range(rows):
        for b in range(K // 16):
            blk = xv[r, 16 * b:16 * b + 16].astype(np.float32)
            q = f32(np.abs(blk).max()) / t
            q = f32(1.0) if q == 0 else q
            q = min(max(q, f32(2.0**-9)), f32(448.0))
            e4 = torch.tensor([float(q)], dtype=torch.float32).to(torch.float8_e4m3fn)
            scales[r, b] = e4.view(torch.uint8).item()
            s = f32(e4.to(torch.float32).item())
            d = s * g
            codes = []
            for v in blk:
                qv = f32(v) / d
                codes.append(e2m1_bruteforce_code(float(qv)) | (8 if v < 0 else 0))
            for j in range(8):
                packed[r, 8 * b + j] = codes[2 * j] | (codes[2 * j + 1] << 4)
    return packed, scales, float(g)


def test_nvfp4_matches_float32_reference():
    x = torch.cat([gen.kv_cache((1, 3, 64)).view(3, 64), gen.mixed_blocks(3, 64),
                   gen.normal_bf16(31, (2, 64))])
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    wp, ws, wg = nvfp4_reference(oracle.decode(bits, "bf16"))
    assert g == wg
    assert np.array_equal(s, ws)
    assert np.array_equal(p, wp)


def test_nvfp4_block_far_below_the_tensor_max_takes_the_smallest_scale():
    # amax_b / (6 g) below 2^-9 clamps to the smallest E4M3 scale 2^-9 (byte
    # 0x01, the page's clamp [2^-9, 448]); the block's values, between
    # 0.25 and 6 grid units of 2^-9 g, still get nonzero codes
    x = torch.zeros(2, 32)
    x[0, 0] = 1.0
    x[0, 1:16] = gen.normal_bf16(41, (15,)).float() * 0.25
    grid = 2.0**-9 / 2688.0
    x[1] = torch.tensor([(0.3 + 0.17 * i) * grid * (-1) ** i for i in range(32)])
    x = x.to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    wp, ws, wg = nvfp4_reference(oracle.decode(bits, "bf16"))
    assert g == wg and np.array_equal(s, ws) and np.array_equal(p, wp)
    assert (s[1] == 0x01).all() and ((p[1] & 0x77) != 0).any()


def test_nvfp4_sign_follows_x_where_the_quotient_underflows():
    # the code's sign bit is taken from x (reading N4): -1e-20 / d underflows
    # to -0.0 in binary32 here (d ~ 448 * 1e30 / 2688) and still gets code 8
    x = torch.zeros(1, 16)
    x[0, 0], x[0, 1], x[0, 2], x[0, 3] = 1e30, -1e-20, -1e-20, 1e-20  # odd and even columns
    bits = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for quantize in (oracle.nvfp4_quantize, oracle.nvfp4_quantize_mse):
        p, s, g = quantize(bits)
        assert (p[0, 0] >> 4) == 8 and (p[0, 1] & 15) == 8 and (p[0, 1] >> 4) == 0


def test_nvfp4_page_facts(facts):
    x = gen.expert_weights(1, 32, 256).view(32, 256).clone()
    x[5, 16:32] = 0.0  # one all-zero block
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    xv = oracle.decode(bits, "bf16")
    amax = np.abs(xv).max()
    assert g == np.float32(np.float32(amax) / np.float32(facts["nvfp4_global_denominator"]))
    decoded = np.array([oracle.decode_e4m3(b) for b in s.reshape(-1)]).reshape(s.shape)
    # the block holding the tensor's largest value gets exactly 448
    r, c = np.unravel_index(np.argmax(np.abs(xv)), xv.shape)
    assert decoded[r, c // 16] == facts["nvfp4_top_block_scale"]
    assert decoded.max() == 448.0 and decoded.min() >= 2.0**-9
    # a zero block takes scale 1.0 and codes 0
    assert decoded[5, 1] == facts["nvfp4_zero_block_scale"]
    assert (p[5, 8:16] == 0).all()
    # 4.5 bits per value: scale bytes are one eighth of packed bytes
    assert s.nbytes * 8 == p.nbytes


def test_nvfp4_dequant_matches_float32_reference():
    x = gen.kv_cache((1, 4, 128)).view(4, 128)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    out = oracle.nvfp4_dequantize(p, s, g, "f32")
    tab = full_table()
    codes = np.stack([p & 15, p >> 4], axis=-1).reshape(4, 128)
    sc = torch.from_numpy(s.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    sc = np.repeat(sc, 16, axis=1)
    want = (tab[codes].astype(np.float32) * sc) * np.float32(g)
    assert np.array_equal(out.view(np.float32), want.astype(np.float32))
    # bf16 output: the binary32 value rounded once more
    outb = oracle.nvfp4_dequantize(p, s, g, "bf16")
    wantb = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(outb, wantb.view(np.uint16))


def test_nvfp4_error_bound():
    # every value lands within half a grid step of its block's scaled grid
    x = gen.expert_weights(1, 16, 512).view(16, 512)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    y = oracle.decode(oracle.nvfp4_dequantize(p, s, g, "f32"), "f32")
    xv = oracle.decode(bits, "bf16")
    sc = np.repeat(np.array([oracle.decode_e4m3(b) for b in s.reshape(-1)]).reshape(s.shape), 16, 1)
    step = sc * g  # one unit of the E2M1 grid in the block; gaps are at most 2 units
    assert (np.abs(y - xv) <= step * 1.0 + 1e-30).all()


def test_nvfp4_zero_tensor():
    bits = np.zeros((2, 32), np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    assert g == 0.0 and (p == 0).all() and (s == 0x38).all()  # 0x38 is E4M3 1.0


# ----------------------------------------------------- packed cache storage

@pytest.mark.parametrize("fmt,B", [("fp8", 128), ("fp8", 32), ("mxfp4", 32), ("nvfp4", 16)])
def test_packed_cache_unpacks_to_the_fake_quantization(fmt, B):
    x = torch.cat([gen.kv_cache((1, 8, 256)).view(8, 256), gen.mixed_blocks(8, 256)])
    bits = x.view(torch.int16).numpy().view(np.uint16)
    codes, scales = oracle.quantize_cache_packed(bits, fmt, B)
    back = oracle.dequantize_cache_packed(codes, scales, fmt, B, 256)
    assert np.array_equal(back, oracle.quantize_cache(bits, fmt, B))


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
def test_packed_cache_scale_bytes_decode_to_the_power_of_two(fmt):
    lo, hi = CLAMP[fmt]
    for k in range(lo, hi + 1):
        b = oracle.cache_scale_byte(k, fmt)
        if fmt == "nvfp4":
            v = torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()
        else:
            v = 2.0 ** (b - 127)
        assert v == 2.0 ** k, (fmt, k, b)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4"])
def test_packed_cache_nan_scale_byte_unpacks_to_nan(fmt):
    # E8M0 byte 0xFF is NaN (reading P2, the E8M0 format): every element of
    # its group unpacks to NaN; the next group is code x 2^(0x7F - 127)
    C, B = 64, 32
    n = C if fmt == "fp8" else C // 2
    codes = ((np.arange(n) * 37 + 5) % 256).astype(np.uint8).reshape(1, n)
    if fmt == "fp8":
        codes[(codes & 0x7F) == 0x7F] = 0x10  # no E4M3 NaN codes
    scales = np.array([[0xFF, 0x7F]], np.uint8)
    v = oracle.decode(oracle.dequantize_cache_packed(codes, scales, fmt, B, C, "f32"), "f32")
    assert np.isnan(v[0, :B]).all()
    if fmt == "fp8":
        want = torch.from_numpy(codes[0, B:].copy()).view(torch.float8_e4m3fn).double().numpy()
    else:
        tail = codes[0, B // 2:]
        want = full_table()[np.stack([tail & 15, tail >> 4], axis=-1).reshape(-1)]
    assert np.array_equal(v[0, B:], want)


def test_packed_cache_codes_follow_the_element_casts():
    x = gen.kv_cache((1, 4, 128)).view(4, 128)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xv = oracle.decode(bits, "bf16")
    codes, scales = oracle.quantize_cache_packed(bits, "fp8", 32)
    ks = scales.astype(int) - 127
    s = np.repeat(2.0 ** ks, 32, axis=1)
    want = torch.from_numpy((xv / s).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(codes, want.view(torch.uint8).numpy())
    c4, s4 = oracle.quantize_cache_packed(bits, "mxfp4", 32)
    k4 = np.repeat(s4.astype(int) - 127, 32, axis=1)
    v = xv / 2.0 ** k4
    nib = np.stack([c4 & 15, c4 >> 4], axis=-1).reshape(4, 128)
    mag = bruteforce_e2m1_mag(np.abs(v).reshape(-1)).reshape(4, 128)
    assert np.array_equal(nib, mag | np.where(xv < 0, 8, 0))


# ----------------------------------------------------- NVFP4 mse block scale

from fractions import Fraction  # noqa: E402

E4M3_VALUE = dict((int(c), float(v)) for v, c in zip(*e4m3_candidates()))


def exact_block_errors(w, g):
    """Exact (rational) squared error of a 16-block for each of the 126
    codes, with the page's binary32 steps done by numpy float32 and the
    E2M1 cast by brute force; None where d underflows to zero."""
    f32 = np.float32
    out = {}
    for c in range(1, 127):
        d = f32(E4M3_VALUE[c]) * f32(g)
        if d == 0:
            out[c] = None
            continue
        v = np.abs(w.astype(np.float32) / d).astype(np.float64)
        q = T8[bruteforce_e2m1_mag(np.minimum(v, 1e30))] * np.where(w < 0, -1.0, 1.0)
        out[c] = sum((Fraction(float(qi)) * Fraction(float(d)) - Fraction(float(wi))) ** 2
                     for qi, wi in zip(q, w))
    return out


def mse_blocks(n_rows=6):
    x = torch.cat([gen.expert_weights(1, n_rows, 64).view(n_rows, 64),
                   gen.mixed_blocks(2, 64), gen.normal_bf16(41, (2, 64))])
    return x.view(torch.int16).numpy().view(np.uint16)


def test_mse_block_error_is_the_exact_sum():
    bits = mse_blocks(2)
    xv = oracle.decode(bits, "bf16")
    g = oracle.nvfp4_global_scale(np.abs(xv).max())
    for w in xv.reshape(-1, 16)[:10]:
        exact = exact_block_errors(w, g)
        for c in (1, 17, 40, 56, 77, 100, 126):
            got = oracle.nvfp4_block_sq_error(w, g, c)
            if exact[c] is None:
                assert got == math.inf
            else:
                # 16 double roundings of a sum of non-negative terms
                assert abs(Fraction(got) - exact[c]) <= exact[c] * Fraction(16, 2**52)


def test_mse_code_is_the_first_exact_minimum():
    bits = mse_blocks()
    xv = oracle.decode(bits, "bf16")
    p, s, g = oracle.nvfp4_quantize_mse(bits)
    assert g == oracle.nvfp4_global_scale(np.abs(xv).max())
    blocks = xv.reshape(-1, 16)
    for b, w in enumerate(blocks):
        exact = {c: e for c, e in exact_block_errors(w, g).items() if e is not None}
        best = min(exact.values())
        c = int(s.reshape(-1)[b])
        slack = best * Fraction(32, 2**52)
        assert exact[c] <= best + slack, b
        # no smaller code is clearly better, nor exactly as good (ties go
        # to the first code)
        assert all(exact[k] > exact[c] - slack for k in exact if k < c), b
        assert not any(exact[k] == exact[c] for k in exact if k < c), b


def test_mse_never_worse_than_the_max_rule():
    bits = mse_blocks()
    xv = oracle.decode(bits, "bf16")
    _, s_mse, g = oracle.nvfp4_quantize_mse(bits)
    _, s_max, g2 = oracle.nvfp4_quantize(bits)
    assert g == g2
    for b, w in enumerate(xv.reshape(-1, 16)):
        e = exact_block_errors(w, g)
        cm, cx = int(s_mse.reshape(-1)[b]), int(s_max.reshape(-1)[b])
        assert e[cm] <= e[cx] * (1 + Fraction(32, 2**52)), b


def test_mse_codes_follow_the_chosen_scale():
    # the packed codes are the max rule's element cast under the chosen scale
    bits = mse_blocks()
    xv = oracle.decode(bits, "bf16")
    p, s, g = oracle.nvfp4_quantize_mse(bits)
    f32 = np.float32
    rows, K = xv.shape
    for r in range(rows):
        for b in range(K // 16):
            d = f32(E4M3_VALUE[int(s[r, b])]) * f32(g)
            for j in range(16):
                v = float(f32(xv[r, 16 * b + j]) / d)
                want = 0 if xv[r, 16 * b + j] == 0 else (
                    e2m1_bruteforce_code(abs(v)) | (8 if xv[r, 16 * b + j] < 0 else 0))
                byte = p[r, 8 * b + j // 2]
                assert (byte >> (4 * (j % 2))) & 15 == want, (r, b, j)


def test_mse_block_on_the_grid_has_zero_error():
    # g = 2^-10 exactly (amax 2.625 = 2688 * 2^-10); a block built as
    # E2M1 values times d = s_c * g for c = 0x30 (1.0) is reconstructed
    # exactly, so the chosen code has zero error
    grid = np.array([6, 4, 3, -2, 1.5, 1, 0.5, 0, -6, -4, 3, 2, -1.5, 1, -0.5, 6])
    d = E4M3_VALUE[0x30] * 2.0**-10
    blk = grid * d
    other = np.zeros(16)
    other[3] = 2.625
    xv = np.stack([np.concatenate([blk, other])])
    bits = torch.from_numpy(xv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.decode(bits, "bf16"), xv)  # exact in bf16
    p, s, g = oracle.nvfp4_quantize_mse(bits)
    assert g == 2.0**-10
    c = int(s[0, 0])
    assert c <= 0x30 and exact_block_errors(xv[0, :16], g)[c] == 0
    assert oracle.nvfp4_block_sq_error(xv[0, :16], g, c) == 0.0


def test_mse_zero_block_and_zero_tensor():
    bits = mse_blocks(1).copy()
    bits[0, 16:32] = 0
    p, s, g = oracle.nvfp4_quantize_mse(bits)
    assert s[0, 1] == 0x01 and (p[0, 8:16] == 0).all()  # every code ties at 0: the first
    p, s, g = oracle.nvfp4_quantize_mse(np.zeros((2, 32), np.uint16))
    assert g == 0.0 and (p == 0).all() and (s == 0x38).all()


def test_mse_moves_codes_both_ways():
    # the page: under the sweep some blocks take a smaller code than the max
    # rule (clipping their largest value) and others a larger one
    x = gen.expert_weights(1, 16, 512).view(16, 512)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    _, s_mse, _ = oracle.nvfp4_quantize_mse(bits)
    _, s_max, _ = oracle.nvfp4_quantize(bits)
    diff = s_mse.astype(int) - s_max.astype(int)
    assert (diff < 0).any() and (diff > 0).any()


# ----------------------------------------------------- W4A4 grouped GEMM

def test_w4a4_matches_numpy_on_quantized_activations():
    # the activations pass through the (pinned) MXFP4 quantizer; the product
    # is then an ordinary matmul with the dequantized weights
    xb, packed, scales, offs = small_moe()
    qp, qs = oracle.mx_quantize(xb, "bf16")
    xq = oracle.decode(oracle.mx_dequantize(qp, qs, "f32"), "f32")
    W = dense_weights(packed, scales)
    want = np.zeros((xb.shape[0], W.shape[1]))
    lo = 0
    for e, hi in enumerate(offs):
        want[lo:hi] = xq[lo:hi] @ W[e].T
        lo = hi
    got = oracle.w4a4_grouped_mm(xb, packed, scales, offs)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_w4a4_differs_from_w4a16_by_the_activation_rounding():
    # quantizing the activations changes the product: the MXFP4 cast moves
    # an element by at most 2 scale units (clipping below 8 to 6, or
    # rounding between 4 and 6) and a unit is at most amax / 4
    xb, packed, scales, offs = small_moe()
    y4 = oracle.w4a4_grouped_mm(xb, packed, scales, offs)
    y16 = oracle.grouped_mm(xb, packed, scales, offs)
    assert not np.allclose(y4, y16)
    W = dense_weights(packed, scales)
    bound = np.abs(oracle.decode(xb, "bf16")).max() / 2 * np.abs(W).sum(axis=2).max()
    assert np.abs(y4 - y16).max() <= bound


def test_w4a4_exact_on_representable_activations():
    # activations already on the MXFP4 grid are left unchanged by the
    # quantizer, so W4A4 equals the bf16-activation GEMM exactly
    xb, packed, scales, offs = small_moe()
    qp, qs = oracle.mx_quantize(xb, "bf16")
    xg = oracle.mx_dequantize(qp, qs, "bf16")
    y4 = oracle.w4a4_grouped_mm(xg, packed, scales, offs)
    y16 = oracle.grouped_mm(xg, packed, scales, offs)
    assert np.array_equal(y4, y16)


# --------------------------------------------- W4A4 NVFP4 grouped GEMM

def nv_dense(packed, bscales, g):
    """float64 values of NVFP4 storage (numpy, from the table and torch's
    E4M3 decode)."""
    tab = full_table()
    codes = np.stack([packed & 15, packed >> 4], axis=-1).reshape(packed.shape[:-1] + (-1,))
    sc = torch.from_numpy(np.ascontiguousarray(bscales)).view(torch.float8_e4m3fn).double().numpy()
    return tab[codes] * np.repeat(sc, 16, axis=-1) * g


def test_nvfp4_quantize_rows_equals_whole_tensor():
    x = torch.cat([gen.kv_cache((1, 3, 64)).view(3, 64), gen.mixed_blocks(3, 64)])
    bits = x.view(torch.int16).numpy().view(np.uint16)
    p, s, g = oracle.nvfp4_quantize(bits)
    p2, s2 = oracle.nvfp4_quantize_rows(bits[2:5], g)
    assert np.array_equal(p2, p[2:5]) and np.array_equal(s2, s[2:5])


def test_nvfp4_w4a4_matches_numpy():
    xb, packed_mx, scales_mx, offs = small_moe()
    E, N = packed_mx.shape[0], packed_mx.shape[1]
    K = 2 * packed_mx.shape[2]
    # NVFP4 weights: each expert quantized as its own tensor
    W = gen.expert_weights(E, N, K).view(torch.int16).numpy().view(np.uint16)
    wp, ws, wg = [], [], []
    for e in range(E):
        p, s, g = oracle.nvfp4_quantize(W[e])
        wp.append(p); ws.append(s); wg.append(g)
    wp, ws, wg = np.stack(wp), np.stack(ws), np.array(wg, np.float32)
    xp, xs, xg = oracle.nvfp4_quantize(xb)
    xq = nv_dense(xp, xs, xg)
    want = np.zeros((xb.shape[0], N))
    lo = 0
    for e, hi in enumerate(offs):
        want[lo:hi] = xq[lo:hi] @ nv_dense(wp[e], ws[e], float(wg[e])).T
        lo = hi
    got = oracle.nvfp4_w4a4_grouped_mm(xb, wp, ws, wg, offs)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
