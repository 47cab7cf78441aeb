"""GPU parity of the W4A4 grouped GEMM (MXFP4 activations x MXFP4 weights
on the block-scaled tensor cores) against the oracle, through the C ABI.

The oracle quantizes the activations with its own MXFP4 quantizer and sums
exactly in double; every product of codes is exact on the tensor core, so
only the f32 accumulation and the final bf16 rounding differ.  Bar:
max |y - ref| / max(|ref|, 1e-2 rms(ref)) <= 1e-2, as for the W4A16 GEMM.
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
TOL = 1e-2


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def error(y, ref):
    y = np.asarray(y, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return np.max(np.abs(y - ref) / np.maximum(np.abs(ref), 1e-2 * rms))


def case(counts, N, K, seed=31, scale_lo=116, scale_hi=124):
    E = len(counts)
    offs = torch.tensor(np.cumsum(counts), dtype=torch.int32)
    T = int(offs[-1])
    packed, scales = gen.random_packed(E, N, K, scale_lo, scale_hi, workload=seed)
    x = gen.normal_bf16(gen.seed_for(seed, 3), (T, K))
    return x, packed, scales, offs


def check(counts, N, K, rows=None, seed=31):
    x, packed, scales, offs = case(counts, N, K, seed)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.w4a4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV), offs.to(DEV),
                            status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    T = x.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ref = oracle.w4a4_grouped_mm(bits(x), packed.numpy(), scales.numpy(), offs.numpy(), rows)
    yv = oracle.decode(bits(y)[rows], "bf16")
    err = error(yv, ref)
    assert err <= TOL, err
    return y


def test_w4a4_small_ragged():
    check([200, 0, 37, 275], 256, 512)


def test_w4a4_many_small_experts_and_one_tile_shapes():
    check([int(c) for c in np.random.RandomState(5).randint(0, 41, size=40)], 128, 256)
    check([1], 128, 256)
    check([300], 384, 768)


def test_w4a4_token_tile_boundaries():
    # N a multiple of 256 takes 224-token tiles: experts of exactly one and
    # two tiles, one token past each, and a single token
    check([224, 225, 448, 449, 1], 256, 512)


def test_w4a4_full_size_sampled():
    # the benchmark GEMM: T=32768, E=32, N=2048, K=7168, multinomial counts
    T, E, N, K = 32768, 32, 2048, 7168
    counts = gen.expert_counts(T, E).numpy()
    offs = torch.tensor(np.cumsum(counts), dtype=torch.int32)
    hp, hs, P, S = full_size_gemm.packed_weights(DEV)  # packed by the oracle
    x = gen.normal_bf16(gen.seed_for(5, 3), (T, K), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.w4a4_grouped_mm(x, P, S, offs.to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = np.array([0, 1, 255, 256, int(offs[0]) - 1, int(offs[0]), 12345, 20000, T - 1])
    ref = oracle.w4a4_grouped_mm(bits(x), hp, hs, offs.numpy(), rows)
    assert error(oracle.decode(bits(y)[rows], "bf16"), ref) <= TOL


def test_w4a4_equals_w4a16_on_grid_activations():
    # activations already on the MXFP4 grid: both GEMMs multiply the same
    # numbers, so they agree within f32 accumulation order
    x, packed, scales, offs = case([130, 126], 256, 512, seed=33)
    xp, xs = mxq.mx_quantize(x.to(DEV))
    xg = mxq.mx_dequantize(xp, xs)
    args = (packed.to(DEV), scales.to(DEV), offs.to(DEV))
    y4 = mxq.w4a4_grouped_mm(xg, *args).float()
    y16 = mxq.mxfp4_grouped_mm(xg, *args).float()
    rel = ((y4 - y16).abs().max() / y16.abs().max()).item()
    assert rel <= 1e-2, rel


def test_w4a4_bad_offs_and_unsupported_shapes():
    x, packed, scales, offs = case([64, 64], 128, 256)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bad = torch.tensor([100, 64], dtype=torch.int32, device=DEV)
    y = torch.full((128, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    mxq.w4a4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV), bad, out=y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -6 and bool((y == 7.0).all())
    x2, p2, s2, o2 = case([64], 128, 96)  # K % 256 != 0
    with pytest.raises(mxq.MxqError) as ei:
        mxq.w4a4_grouped_mm(x2.to(DEV), p2.to(DEV), s2.to(DEV), o2.to(DEV))
    assert ei.value.status == -4


# ---------------------------------------------------------------- NVFP4

def nv_weights(E, N, K, seed=41):
    """Random NVFP4 weight storage from the seeded generator: code bytes,
    E4M3 block-scale bytes in [0x30, 0x40] (0.5 .. 2.0) and per-expert
    global scales."""
    packed = gen.random_bytes(E * N * (K // 2), gen.seed_for(seed, 1)).view(E, N, K // 2)
    u = gen.uniform(gen.seed_for(seed, 2), E * N * (K // 16))
    bs = (u * 17).floor().clamp_(max=16).to(torch.uint8).add_(0x30).view(E, N, K // 16)
    gw = torch.tensor([0.01 * (1 + e / E) for e in range(E)], dtype=torch.float32)
    return packed, bs, gw


def nv_check(counts, N, K, rows=None, seed=41):
    E = len(counts)
    offs = torch.tensor(np.cumsum(counts), dtype=torch.int32)
    T = int(offs[-1])
    packed, bs, gw = nv_weights(E, N, K, seed)
    x = gen.normal_bf16(gen.seed_for(seed, 3), (T, K))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.nvfp4_w4a4_grouped_mm(x.to(DEV), packed.to(DEV), bs.to(DEV), gw.to(DEV),
                                  offs.to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ref = oracle.nvfp4_w4a4_grouped_mm(bits(x), packed.numpy(), bs.numpy(), gw.numpy(),
                                       offs.numpy(), rows)
    err = error(oracle.decode(bits(y)[rows], "bf16"), ref)
    assert err <= TOL, err


def test_nvfp4_w4a4_small_ragged():
    nv_check([200, 0, 37, 275], 256, 512)


def test_nvfp4_w4a4_many_small_experts():
    nv_check([int(c) for c in np.random.RandomState(7).randint(0, 41, size=24)], 128, 256)
    nv_check([300], 384, 768)


def test_nvfp4_w4a4_token_tile_boundaries():
    nv_check([224, 225, 448, 449, 1], 256, 512)


def test_nvfp4_w4a4_full_size_sampled():
    T, E, N, K = 32768, 32, 2048, 7168
    counts = gen.expert_counts(T, E).numpy()
    rows = [0, 1, 255, 256, int(np.cumsum(counts)[0]), 20000, T - 1]
    nv_check(list(counts), N, K, rows=rows)


def test_prequantized_activations_give_the_same_bits():
    # x_quantized: the block-scaled GEMM alone on activations quantized beforehand
    counts = [200, 0, 37, 275]
    x, packed, scales, offs = case(counts, 256, 512)
    xd, pd, sd, od = x.to(DEV), packed.to(DEV), scales.to(DEV), offs.to(DEV)
    want = mxq.w4a4_grouped_mm(xd, pd, sd, od)
    xq, xs = mxq.mx_quantize(xd)
    got = mxq.w4a4_grouped_mm(None, pd, sd, od, x_quantized=(xq, xs))
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    wn = gen.expert_weights(len(counts), 256, 512).view(torch.int16).numpy().view(np.uint16)
    qs = [oracle.nvfp4_quantize(wn[e]) for e in range(len(counts))]
    nvp = torch.from_numpy(np.stack([q[0] for q in qs])).to(DEV)
    nvs = torch.from_numpy(np.stack([q[1] for q in qs])).to(DEV)
    nvg = torch.tensor([q[2] for q in qs], dtype=torch.float32, device=DEV)
    want = mxq.nvfp4_w4a4_grouped_mm(xd, nvp, nvs, nvg, od)
    got = mxq.nvfp4_w4a4_grouped_mm(None, nvp, nvs, nvg, od,
                                    x_quantized=mxq.nvfp4_quantize(xd))
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    # wrong operand shapes are refused before a launch
    with pytest.raises(ValueError, match="x_quantized"):
        mxq.w4a4_grouped_mm(None, pd, sd, od, x_quantized=(xq[:, :-1], xs))
    with pytest.raises(ValueError, match="x_quantized"):
        mxq.w4a4_grouped_mm(None, pd, sd, od, x_quantized=(xq, xs[:-1]))

