"""Seeded synthetic inputs for the tests and the benchmark.

This module only draws random numbers; it holds none of the quantization
arithmetic.  Every draw comes from one counter-based generator, SplitMix64
(Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014): the i-th 64-bit output for a seed is a pure function of
(seed, i), evaluated with wrapping int64 tensor arithmetic, so the same call
gives the same numbers on the CPU and on a GPU.  Normal deviates use the
Box-Muller transform in float64 and are then rounded to the element dtype by
torch's own cast; the tests always hand the oracle the very bytes the GPU
sees (copied back), so host/device libm differences cannot matter.

Seeds follow ``20261202 + 100 * workload + tensor_index``.
"""
import math

import torch

_GOLDEN = 0x9E3779B97F4A7C15 - (1 << 64)
_M1 = 0xBF58476D1CE4E5B9 - (1 << 64)
_M2 = 0x94D049BB133111EB - (1 << 64)
_CHUNK = 1 << 25


def seed_for(workload: int, tensor_index: int) -> int:
    return 20261202 + 100 * workload + tensor_index


def _srl(z, s):
    """Logical right shift of int64 lanes."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(seed: int, start: int, n: int, device) -> torch.Tensor:
    """Outputs start .. start+n-1 of SplitMix64(seed) as int64 lanes."""
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = i * _GOLDEN + (seed & ((1 << 63) - 1))
    z = (z ^ _srl(z, 30)) * _M1
    z = (z ^ _srl(z, 27)) * _M2
    return z ^ _srl(z, 31)


def uniform(seed: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """float64 in [0, 1): the top 53 bits of each output."""
    return _srl(splitmix64(seed, start, n, device), 11).to(torch.float64) * (2.0 ** -53)


def normal(seed: int, n: int, device="cpu") -> torch.Tensor:
    """float64 N(0, 1) by Box-Muller on consecutive output pairs."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        m = min(_CHUNK, n - c0)
        u = uniform(seed, 2 * m, device, start=2 * c0).view(m, 2)
        u1 = 1.0 - u[:, 0]  # (0, 1]
        r = torch.sqrt(-2.0 * torch.log(u1))
        out[c0:c0 + m] = r * torch.cos((2.0 * math.pi) * u[:, 1])
    return out


def normal_bf16(seed: int, shape, std: float = 1.0, device="cpu") -> torch.Tensor:
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for c0 in range(0, n, _CHUNK):
        m = min(_CHUNK, n - c0)
        # Chunks draw disjoint counter ranges: offset the seed's stream by c0.
        u = uniform(seed, 2 * m, device, start=2 * c0).view(m, 2)
        r = torch.sqrt(-2.0 * torch.log(1.0 - u[:, 0]))
        out[c0:c0 + m] = (std * r * torch.cos((2.0 * math.pi) * u[:, 1])).to(torch.bfloat16)
    return out.view(*shape)


# ---- the workloads ---------------------------------------------------------

def mx_small(device="cpu") -> torch.Tensor:
    """bf16 [64, 256] ~ N(0,1) with four forced rows:
    row 0 all zero; row 1 all 1.75; row 2 with every 32-block's largest
    magnitude exactly 2.0 (one element +-2, the rest kept below 2); row 3 all
    2^-3."""
    x = normal_bf16(seed_for(1, 0), (64, 256), device=device)
    x[0] = 0.0
    x[1] = 1.75
    row = x[2].float().clamp(-1.984375, 1.984375)
    sign = torch.where(uniform(seed_for(1, 1), 8, device) < 0.5, -2.0, 2.0).to(row.dtype)
    pos = (uniform(seed_for(1, 2), 8, device) * 32).long()
    for b in range(8):
        row[b * 32 + int(pos[b])] = sign[b]
    x[2] = row.to(torch.bfloat16)
    x[3] = 0.125
    return x


def kv_cache(shape=(4, 8192, 512), device="cpu", seed_base: int = 0) -> torch.Tensor:
    """bf16 KV-cache-like activations: N(0,1) times a per-channel scale
    10^U(-3, 2) (shared over the leading dims), with 0.1% of entries (uniform
    positions) multiplied by +-100."""
    C = shape[-1]
    n = math.prod(shape)
    ch = torch.pow(10.0, -3.0 + 5.0 * uniform(seed_for(2, 10 + seed_base), C, device))
    z = normal(seed_for(2, 0 + seed_base), n, device).view(-1, C) * ch
    z = z.view(-1)
    u = uniform(seed_for(2, 1 + seed_base), n, device)
    hit = u < 1e-3
    sgn = torch.where(uniform(seed_for(2, 2 + seed_base), n, device) < 0.5, -100.0, 100.0)
    z = torch.where(hit, z * sgn, z)
    return z.to(torch.bfloat16).view(*shape)


def expert_weights(E=64, N=2048, K=7168, std=0.02, device="cpu", workload=3) -> torch.Tensor:
    """bf16 [E, N, K] ~ N(0, std^2)."""
    return normal_bf16(seed_for(workload, 0), (E, N, K), std=std, device=device)


def mixed_blocks(R, C=7168, device="cpu") -> torch.Tensor:
    """bf16 [R, C]; every 32-column block is independently one of: normal
    N(0,1) (85%), subnormal-range N(0,1)*1e-40 (5%), all zero (5%), or a
    single spike (5%: 31 values N(0,1)*1e-2 and one +-64*(1+U))."""
    assert C % 32 == 0
    n = R * C
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    step = _CHUNK
    for c0 in range(0, n, step):
        m = min(step, n - c0)
        b0, nb = c0 // 32, m // 32
        z = _normal_range(seed_for(4, 1), c0, m, device)
        kind_u = uniform(seed_for(4, 0), nb, device, start=b0)
        kind = (kind_u >= 0.85).to(torch.int8) + (kind_u >= 0.90) + (kind_u >= 0.95)
        k = kind.repeat_interleave(32)
        spike_pos = (uniform(seed_for(4, 2), nb, device, start=b0) * 32).long()
        spike_val = 64.0 * (1.0 + uniform(seed_for(4, 3), nb, device, start=b0))
        spike_sgn = torch.where(uniform(seed_for(4, 4), nb, device, start=b0) < 0.5, -1.0, 1.0)
        lane = torch.arange(m, device=device) % 32
        at_pos = lane == spike_pos.repeat_interleave(32)
        spike = (spike_val * spike_sgn).repeat_interleave(32)
        z = torch.where(k == 1, z * 1e-40, z)
        z = torch.where(k == 2, torch.zeros_like(z), z)
        z = torch.where((k == 3) & at_pos, spike, torch.where(k == 3, z * 1e-2, z))
        out[c0:c0 + m] = z.to(torch.bfloat16)
    return out.view(R, C)


def _normal_range(seed, start, m, device):
    u = uniform(seed, 2 * m, device, start=2 * start).view(m, 2)
    r = torch.sqrt(-2.0 * torch.log(1.0 - u[:, 0]))
    return r * torch.cos((2.0 * math.pi) * u[:, 1])


def expert_counts(T=32768, E=32, device="cpu", seed=None) -> torch.Tensor:
    """Row counts per expert: a seeded multinomial of T draws over E equally
    likely experts (each token draws its expert uniformly)."""
    s = seed_for(5, 2) if seed is None else seed
    ids = (uniform(s, T, device) * E).long().clamp_(max=E - 1)
    return torch.bincount(ids, minlength=E)


def random_packed(E, N, K, scale_lo=110, scale_hi=130, device="cpu", workload=5):
    """Random MXFP4 storage: uniformly random code bytes [E, N, K/2] and
    scale bytes uniform in [scale_lo, scale_hi] ([E, N, K/32])."""
    nb = E * N * (K // 2)
    ns = E * N * (K // 32)
    packed = (_srl(splitmix64(seed_for(workload, 7), 0, nb, device), 56)).to(torch.uint8)
    sc = uniform(seed_for(workload, 8), ns, device) * (scale_hi - scale_lo + 1) + scale_lo
    scales = sc.floor().clamp_(max=scale_hi).to(torch.uint8)
    return packed.view(E, N, K // 2), scales.view(E, N, K // 32)


def random_bytes(n, seed, device="cpu") -> torch.Tensor:
    return _srl(splitmix64(seed, 0, n, device), 56).to(torch.uint8)
