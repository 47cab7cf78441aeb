"""GPU parity of NVFP4 quantization with mse block scales (the sweep over
the 126 positive finite E4M3 codes), through the C ABI.

Codes, block-scale bytes and the per-tensor scale must equal the oracle's
bit for bit: the oracle takes every decision in the same arithmetic as the
kernel (binary32 quotients, exact double errors summed in element order),
so there is no tolerance.  At the full expert-weight size, sampled rows are
compared with the oracle and every block is checked to reconstruct with no
more squared error than the max rule's scale.
"""
import numpy as np
import pytest
import torch

import nvfp4_quantization_amax_b200 as mxq
import oracle
import synthetic as gen

pytestmark = pytest.mark.gpu

DEV = "cuda"
_NP = {torch.bfloat16: np.uint16, torch.float16: np.uint16, torch.float32: np.uint32}
_INT = {torch.bfloat16: torch.int16, torch.float16: torch.int16, torch.float32: torch.int32}
_NAME = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}


def bits(t):
    return t.detach().cpu().contiguous().view(_INT[t.dtype]).numpy().view(_NP[t.dtype])


def u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def assert_equal(got, want, what):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got.reshape(-1) != want.reshape(-1))[0]
    assert bad.size == 0, "%s: %d mismatches, first at %s: got %s want %s" % (
        what, bad.size, bad[:4], got.reshape(-1)[bad[:4]], want.reshape(-1)[bad[:4]])


def check(x, dtype_name="bf16"):
    p, s, g = mxq.nvfp4_quantize(x, rule="mse")
    wp, ws, wg = oracle.nvfp4_quantize_mse(bits(x), dtype_name)
    assert float(g.item()) == wg
    assert_equal(u8(s), ws, "block scales")
    assert_equal(u8(p), wp, "packed")
    return p, s, g


def test_mse_expert_weight_rows_exact():
    check(gen.expert_weights(1, 96, 2048, device=DEV).view(96, 2048))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_mse_dtypes_and_mixed_blocks_exact(dtype):
    x = torch.cat([gen.mixed_blocks(32, 512), gen.kv_cache((1, 16, 512)).view(16, 512)])
    x = x.to(dtype)
    if dtype == torch.float32:
        x[:8] *= torch.logspace(-20, 20, 512, dtype=torch.float64).float()
    check(x.to(DEV), _NAME[dtype])


def test_mse_zero_blocks_ragged_and_zero_tensor():
    x = gen.normal_bf16(78, (5, 48))
    x[2, 16:32] = 0.0
    x[3, 0:16] = -0.0
    p, s, g = check(x.to(DEV))  # 15 blocks: a partial group of lanes at the end
    assert int(s[2, 1]) == 0x01 and int(s[3, 0]) == 0x01
    z = torch.zeros(3, 48, dtype=torch.bfloat16, device=DEV)
    p, s, g = mxq.nvfp4_quantize(z, rule="mse")
    assert float(g.item()) == 0.0 and int(p.max()) == 0 and bool((s == 0x38).all())


def block_sq_error(x, p, s, g):
    """Per-block squared error of the NVFP4 reconstruction, in float64."""
    y = mxq.nvfp4_dequantize(p, s, g, torch.float32).double()
    return ((y - x.double()) ** 2).view(-1, 16).sum(dim=1)


def test_mse_full_expert_weight():
    x = gen.expert_weights(1, 2048, 7168, device=DEV).view(2048, 7168)
    p, s, g = mxq.nvfp4_quantize(x, rule="mse")
    xb = bits(x)
    wg = oracle.nvfp4_global_scale(np.abs(oracle.decode(xb, "bf16")).max())
    assert float(g.item()) == wg
    # the first and last row and 128 seeded ones (oracle rows on all host cores)
    rows = np.unique(np.concatenate([[0, 2047], np.random.RandomState(11).choice(2048, 128, replace=False)]))
    with oracle.all_cores():
        wp, ws, _ = oracle.nvfp4_quantize_mse(xb[rows], g=wg)
    assert_equal(u8(s[torch.from_numpy(rows).to(DEV)]), ws, "sampled scales")
    assert_equal(u8(p[torch.from_numpy(rows).to(DEV)]), wp, "sampled packed")
    # every block: no worse than the max rule (the dequantized product rounds
    # once in binary32, hence the small slack)
    pm, sm, gm = mxq.nvfp4_quantize(x)
    e_mse, e_max = block_sq_error(x, p, s, g), block_sq_error(x, pm, sm, gm)
    energy = (x.double() ** 2).view(-1, 16).sum(dim=1)
    assert bool((e_mse <= e_max * (1 + 1e-6) + 1e-12 * energy).all())
    assert float(e_mse.sum()) < float(e_max.sum())


def test_mse_ties_and_pruning_edges():
    # blocks where many scale codes tie (a single nonzero weight, constant
    # blocks, values on the E2M1 grid) and blocks whose weights are tiny or
    # huge next to the tensor maximum (the top and bottom of the code range)
    rows = []
    vals = [2.0 ** k for k in range(-12, 6)] + [3.0, 0.75, 1.5, 6.0, 0.1, 7.0]
    for v in vals:
        b = np.zeros(16)
        b[5] = v
        rows.append(b)
        rows.append(np.full(16, v))
        rows.append(np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 0.0]) * v)
    x = torch.tensor(np.concatenate(rows).reshape(-1, 64), dtype=torch.float32)
    x[0, 0] = 2000.0  # the tensor maximum: small blocks sit near the bottom codes
    for dtype in (torch.bfloat16, torch.float32):
        xd = x.to(dtype)
        check(xd.to(DEV), "bf16" if dtype == torch.bfloat16 else "f32")
