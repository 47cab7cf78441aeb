"""GPU parity of the grouped GEMMs at the edges of the weight decode.

Every scale byte a weight can carry (0 .. 252, where W_e is exact in bf16;
"nemo_automodel.components.quantization.mxfp4", dequantize_mxfp4 and
MXFP4GroupedMM) is fed through the tensor-core paths: experts whose weights
decode to bf16 subnormals (scale bytes 0..7), to the largest finite weights
(bytes up to 252), weights packed by mx_quantize from the mixed-block
workload (zero, subnormal-range and single-spike 32-blocks), and bf16
subnormal activations.  Each expert's activation rows are scaled by a power
of two so that its products stay finite.

Bar, per expert e (rows the expert owns, rms over those rows of the exact
sum):  |y - ref| <= 1e-2 * max(|ref|, 1e-2 * rms_e) + 2^-133.
The relative part is the bound fixed for this path; taking the rms per
expert keeps an expert of tiny outputs from hiding under its neighbours'.
The absolute 2^-133 is one spacing of the bf16 subnormals: y is rounded to
bf16, so where |ref| < 2^-126 no result can be closer than half a spacing,
and the f32 accumulation may push it across one rounding boundary.  It
matters only for outputs below ~1e-38.
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
REL = 1e-2
ABS = 2.0 ** -133

# (scale byte lo, hi, log2 of the activation scale, activation kind)
EXPERTS = [
    (0, 7, 124, "normal"),      # bf16-subnormal weights x large activations: normal products
    (0, 7, 0, "normal"),        # bf16-subnormal weights x N(0,1): f32-subnormal products
    (8, 60, 93, "normal"),
    (61, 115, 39, "normal"),
    (116, 150, 0, "normal"),
    (151, 180, -38, "normal"),
    (181, 210, -68, "normal"),
    (211, 240, -98, "normal"),
    (241, 252, -119, "normal"),  # the largest finite weights
    (None, None, 0, "normal"),   # weights packed by mx_quantize from mixed blocks
    (116, 124, 0, "subnormal"),  # bf16-subnormal activations x normal weights
    (240, 252, 0, "subnormal"),  # bf16-subnormal activations x large weights
    (116, 124, 0, "empty"),      # an expert without rows
]
ROWS = [70, 33, 64, 1, 90, 47, 130, 65, 40, 100, 64, 71, 0]


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def edge_weights(N, K, seed):
    """Packed [E, N, K/2] and scales [E, N, K/32], one scale-byte range per
    expert; the mixed-block expert is packed by the oracle's quantizer."""
    ps, ss = [], []
    for e, (lo, hi, _, _) in enumerate(EXPERTS):
        if lo is None:
            w = gen.mixed_blocks(N, K)
            p, s = oracle.mx_quantize(bits(w))
            p, s = torch.from_numpy(p).view(1, N, K // 2), torch.from_numpy(s).view(1, N, K // 32)
        else:
            p, s = gen.random_packed(1, N, K, lo, hi, workload=seed + e)
        ps.append(p)
        ss.append(s)
    return torch.cat(ps).contiguous(), torch.cat(ss).contiguous()


def edge_activations(cols, seed):
    """bf16 [T, cols]: each expert's rows N(0,1) times 2^shift, or bf16
    subnormals N(0,1)*1e-40."""
    parts = []
    for e, ((_, _, shift, kind), n) in enumerate(zip(EXPERTS, ROWS)):
        if n == 0:
            continue
        z = gen.normal_bf16(gen.seed_for(seed, 20 + e), (n, cols)).float()
        z = z * 1e-40 if kind == "subnormal" else z * 2.0 ** shift
        parts.append(z.to(torch.bfloat16))
    return torch.cat(parts)


def owners(offs, rows):
    return np.searchsorted(np.asarray(offs), np.asarray(rows), side="right")


def assert_per_expert(y, ref, owner, what):
    y = np.asarray(y, np.float64)
    assert np.all(np.isfinite(ref)), what
    worst = 0.0
    for e in np.unique(owner):
        m = owner == e
        r = ref[m]
        rms = np.sqrt(np.mean(r ** 2))
        bound = REL * np.maximum(np.abs(r), 1e-2 * rms) + ABS
        excess = np.abs(y[m] - r) / bound
        i = int(np.argmax(excess))  # index into the flattened outputs
        assert excess.flat[i] <= 1.0, "%s: expert %d output %d: got %r want %r (rms %r)" % (
            what, e, i, y[m].flat[i], r.flat[i], rms)
        worst = max(worst, float(excess.flat[i]))
    return worst


def run_edges(N, K, transpose_w, seed=61):
    packed, scales = edge_weights(N, K, seed)
    offs = np.cumsum(ROWS).astype(np.int32)
    a = edge_activations(N if transpose_w else K, seed)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a.to(DEV), packed.to(DEV), scales.to(DEV),
                             torch.from_numpy(offs).to(DEV), transpose_w=transpose_w,
                             status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.grouped_mm(bits(a), packed.numpy(), scales.numpy(), offs,
                            transpose_w=transpose_w)
    rows = np.arange(a.shape[0])
    yv = oracle.decode(bits(y), "bf16")
    return assert_per_expert(yv, ref, owners(offs, rows), "N=%d K=%d t=%d" % (N, K, transpose_w))


@pytest.mark.parametrize("transpose_w", [False, True])
@pytest.mark.parametrize("N,K", [(256, 512),   # CTA-pair tiles both ways
                                 (128, 384),   # single-CTA tiles both ways
                                 (100, 96)])   # the general kernel
def test_grouped_mm_every_scale_byte_range(N, K, transpose_w):
    run_edges(N, K, transpose_w)


def test_edge_weights_cover_the_decode_range():
    # the cases above really carry what they claim: scale bytes 0 and 252,
    # nonzero codes under byte 0 (bf16-subnormal weights), and the zero /
    # subnormal-range / spike blocks of the mixed workload
    packed, scales = edge_weights(256, 512, 61)
    s = scales.numpy()
    assert s.min() == 0 and s.max() == 252
    w0 = oracle.mx_dequantize(packed[0].numpy(), scales[0].numpy(), "f32")
    v0 = oracle.decode(w0, "f32")
    nz = v0[v0 != 0]
    assert nz.size > 0 and np.abs(nz).max() <= 6 * 2.0 ** -120  # byte 7 at most
    assert np.any(np.abs(nz) < 2.0 ** -126)
    mixed = s[9]
    assert (mixed == 0).any() and (mixed >= 130).any()
    x = edge_activations(512, 61).float()
    sub = x[sum(ROWS[:10]):sum(ROWS[:11])]
    assert bool((sub.abs() < 2.0 ** -126).all()) and bool((sub != 0).any())


# ---------------------------------------------------- full size, sampled

def sampled_rows(offs, per_expert=16, seed=8):
    """Every expert's first and last row plus `per_expert` seeded rows."""
    rng = np.random.default_rng(seed)
    starts = np.concatenate([[0], offs[:-1]])
    rows = []
    for lo, hi in zip(starts, offs):
        if hi > lo:
            rows += [lo, hi - 1] + list(rng.integers(lo, hi, per_expert))
    return np.unique(np.array(rows, np.int64))


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_full_size_eighteen_rows_per_expert(transpose_w):
    T, E, N, K = 32768, 32, 2048, 7168
    counts = gen.expert_counts(T, E).numpy()
    offs = np.cumsum(counts).astype(np.int32)
    rows = sampled_rows(offs)
    hp, hs, packed, scales = full_size_gemm.packed_weights(DEV)  # packed by the oracle
    a = gen.normal_bf16(gen.seed_for(5, 4 if transpose_w else 3), (T, N if transpose_w else K),
                        device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a, packed, scales, torch.from_numpy(offs).to(DEV),
                             transpose_w=transpose_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.grouped_mm(bits(a), packed.cpu().numpy(), scales.cpu().numpy(), offs,
                            transpose_w=transpose_w, rows=rows)
    yv = oracle.decode(bits(y[torch.from_numpy(rows).to(DEV)]), "bf16")
    assert_per_expert(yv, ref, owners(offs, rows), "full size t=%d" % transpose_w)


# ------------------------------------------------------------ W4A4 (MXFP4)

# activation scale (log2) per expert chosen so that the MXFP4 activation
# scale byte sits at the other end of the range from the weight's
W4_EXPERTS = [(0, 7, 124), (8, 60, 93), (116, 124, 0), (151, 180, -38), (241, 252, -119),
              (116, 124, -126), (0, 7, 0)]
W4_ROWS = [70, 1, 129, 64, 40, 33, 50]


def test_w4a4_every_scale_byte_range():
    N, K = 256, 512
    ps, ss, xs = [], [], []
    for e, ((lo, hi, shift), n) in enumerate(zip(W4_EXPERTS, W4_ROWS)):
        p, s = gen.random_packed(1, N, K, lo, hi, workload=71 + e)
        ps.append(p)
        ss.append(s)
        z = gen.normal_bf16(gen.seed_for(71, 30 + e), (n, K)).float() * 2.0 ** shift
        xs.append(z.to(torch.bfloat16))
    packed, scales = torch.cat(ps), torch.cat(ss)
    x = torch.cat(xs)
    offs = np.cumsum(W4_ROWS).astype(np.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.w4a4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV),
                            torch.from_numpy(offs).to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = np.arange(x.shape[0])
    ref = oracle.w4a4_grouped_mm(bits(x), packed.numpy(), scales.numpy(), offs, rows)
    assert_per_expert(oracle.decode(bits(y), "bf16"), ref, owners(offs, rows), "w4a4 edges")


def test_w4a4_mixed_block_activations_and_weights():
    # activations and weights from the mixed-block workload: zero blocks
    # (activation scale byte 0), subnormal-range blocks and spikes
    N, K, counts = 256, 512, [90, 0, 166]
    E = len(counts)
    w = gen.mixed_blocks(E * N, K)
    p, s = oracle.mx_quantize(bits(w))
    packed = torch.from_numpy(p).view(E, N, K // 2)
    scales = torch.from_numpy(s).view(E, N, K // 32)
    x = gen.mixed_blocks(sum(counts), K)
    offs = np.cumsum(counts).astype(np.int32)
    y = mxq.w4a4_grouped_mm(x.to(DEV), packed.to(DEV), scales.to(DEV),
                            torch.from_numpy(offs).to(DEV))
    torch.cuda.synchronize()
    rows = np.arange(x.shape[0])
    ref = oracle.w4a4_grouped_mm(bits(x), p.reshape(E, N, K // 2), s.reshape(E, N, K // 32),
                                 offs, rows)
    assert_per_expert(oracle.decode(bits(y), "bf16"), ref, owners(offs, rows), "w4a4 mixed")


def test_w4a4_full_size_eighteen_rows_per_expert():
    T, E, N, K = 32768, 32, 2048, 7168
    counts = gen.expert_counts(T, E).numpy()
    offs = np.cumsum(counts).astype(np.int32)
    rows = sampled_rows(offs)
    hp, hs, P, S = full_size_gemm.packed_weights(DEV)  # packed by the oracle
    x = gen.normal_bf16(gen.seed_for(5, 3), (T, K), device=DEV)
    y = mxq.w4a4_grouped_mm(x, P, S, torch.from_numpy(offs).to(DEV))
    torch.cuda.synchronize()
    ref = oracle.w4a4_grouped_mm(bits(x), hp, hs, offs, rows)
    yv = oracle.decode(bits(y[torch.from_numpy(rows).to(DEV)]), "bf16")
    assert_per_expert(yv, ref, owners(offs, rows), "w4a4 full size")


# ------------------------------------------------------------ W4A4 (NVFP4)

def test_nvfp4_w4a4_global_scales_far_apart():
    # experts whose NVFP4 weights differ by up to 2^200 in magnitude: the
    # product of the two global scales runs from ~2^-119 to ~2^81
    N, K, counts = 256, 512, [64, 37, 100, 1, 80]
    mags = [2.0 ** -100, 2.0 ** -40, 1.0, 2.0 ** 40, 2.0 ** 100]
    ps, bss, gws = [], [], []
    for e, m in enumerate(mags):
        w = (gen.normal_bf16(gen.seed_for(81, e), (N, K)).float() * m).to(torch.bfloat16)
        p, bs, g = oracle.nvfp4_quantize(bits(w))
        ps.append(torch.from_numpy(p).view(1, N, K // 2))
        bss.append(torch.from_numpy(bs).view(1, N, K // 16))
        gws.append(g)
    packed, bs = torch.cat(ps), torch.cat(bss)
    gw = torch.tensor(gws, dtype=torch.float32)
    x = gen.normal_bf16(gen.seed_for(81, 10), (sum(counts), K))
    offs = np.cumsum(counts).astype(np.int32)
    y = mxq.nvfp4_w4a4_grouped_mm(x.to(DEV), packed.to(DEV), bs.to(DEV), gw.to(DEV),
                                  torch.from_numpy(offs).to(DEV))
    torch.cuda.synchronize()
    rows = np.arange(x.shape[0])
    ref = oracle.nvfp4_w4a4_grouped_mm(bits(x), packed.numpy(), bs.numpy(), gw.numpy(), offs,
                                       rows)
    assert_per_expert(oracle.decode(bits(y), "bf16"), ref, owners(offs, rows), "nvfp4 w4a4")


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_reduced_benchmark_case_all_outputs(transpose_w):
    # the benchmark workload's recipe at T=4096, E=8, N=256, K=512: every
    # output against the oracle's exact sum, weights packed by the oracle
    T, E, N, K = 4096, 8, 256, 512
    offs = np.cumsum(gen.expert_counts(T, E).numpy()).astype(np.int32)
    W = gen.expert_weights(E, N, K, workload=5)
    packed, scales = oracle.mx_quantize(bits(W).reshape(E * N, K), "bf16")
    packed, scales = packed.reshape(E, N, K // 2), scales.reshape(E, N, K // 32)
    a = gen.normal_bf16(gen.seed_for(5, 4 if transpose_w else 3), (T, N if transpose_w else K))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a.to(DEV), torch.from_numpy(packed).to(DEV),
                             torch.from_numpy(scales).to(DEV), torch.from_numpy(offs).to(DEV),
                             transpose_w=transpose_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    with oracle.all_cores():
        ref = oracle.grouped_mm(bits(a), packed, scales, offs, transpose_w=transpose_w)
    rows = np.arange(T)
    assert_per_expert(oracle.decode(bits(y), "bf16"), ref, owners(offs, rows), "reduced case")


@pytest.mark.parametrize("transpose_w", [False, True])
def test_grouped_mm_full_size_all_outputs_against_fp32_matmul(transpose_w):
    # A secondary check, beside the oracle's sampled rows: every output of
    # the benchmark GEMM against an fp32 matrix product (torch, TF32 off)
    # per expert, of the weights the oracle dequantizes.  The product's own
    # error (fp32 accumulation over <= 7168 terms) is far inside the bar.
    T, E, N, K = full_size_gemm.T, full_size_gemm.E, full_size_gemm.N, full_size_gemm.K
    hp, hs, packed, scales = full_size_gemm.packed_weights(DEV)
    offs = full_size_gemm.offsets()
    a = gen.normal_bf16(gen.seed_for(5, 4 if transpose_w else 3), (T, N if transpose_w else K),
                        device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mxq.mxfp4_grouped_mm(a, packed, scales, torch.from_numpy(offs).to(DEV),
                             transpose_w=transpose_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    with oracle.all_cores():
        wbits = oracle.mx_dequantize(hp, hs, "bf16")  # [E, N, K] bf16 bits
    W = torch.from_numpy(wbits.view(np.int16)).to(DEV).view(torch.bfloat16)
    del wbits
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        worst = 0.0
        lo = 0
        for e in range(E):
            hi = int(offs[e])
            if hi == lo:
                continue
            We = W[e].float()
            ref = a[lo:hi].float() @ (We if transpose_w else We.t())
            got = y[lo:hi].float()
            rms = ref.pow(2).mean().sqrt()
            bound = REL * torch.maximum(ref.abs(), 1e-2 * rms) + ABS
            excess = float(((got - ref).abs() / bound).max())
            assert excess <= 1.0, "expert %d: %r" % (e, excess)
            worst = max(worst, excess)
            lo = hi
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
