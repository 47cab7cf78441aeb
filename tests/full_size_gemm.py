"""The benchmark grouped-GEMM workload for the parity tests: T=32768 tokens,
E=32 experts, N=2048, K=7168, multinomial expert counts, expert weights
N(0, 0.02^2) packed to MXFP4 by the oracle.  The packed bytes the GPU
multiplies are the oracle's own, so no input of the oracle comes from the
GPU path."""
import functools

import numpy as np
import torch

import oracle
import synthetic as gen

T, E, N, K = 32768, 32, 2048, 7168


@functools.lru_cache(maxsize=1)
def _oracle_packed():
    W = gen.expert_weights(E, N, K, device="cuda", workload=5)
    bits = W.view(torch.int16).cpu().numpy().view(np.uint16).reshape(E * N, K)
    del W
    with oracle.all_cores():
        p, s = oracle.mx_quantize(bits, "bf16")
    return p.reshape(E, N, K // 2), s.reshape(E, N, K // 32)


def packed_weights(device="cuda"):
    """(packed [E, N, K/2], scales [E, N, K/32]) uint8: host numpy arrays
    and their device copies."""
    p, s = _oracle_packed()
    return p, s, torch.from_numpy(p).to(device), torch.from_numpy(s).to(device)


def offsets():
    """int32 [E]: inclusive prefix sums of the seeded multinomial counts."""
    return np.cumsum(gen.expert_counts(T, E).numpy()).astype(np.int32)
