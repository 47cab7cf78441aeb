"""GPU parity of the stored cache form (codes + scale bytes) and of the
straight-through CacheQuantization function, through the C ABI.

Codes and scale bytes must equal the oracle's byte for byte, the unpacked
values must equal the oracle's unpack bit for bit, and unpack(pack(x)) must
equal the fake quantization quantize_cache(x) bit for bit (a property that
holds at any size, so it is checked on the full KV-cache workload too).
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
FORMATS = [("fp8", 128), ("mxfp4", 32), ("nvfp4", 16)]


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


def to_float(b, dtype):
    """float32 values of raw bf16 / f32 bit patterns."""
    if dtype == torch.float32:
        return b.view(np.float32)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()


def check_case(x, fmt, B, dtype_name="bf16"):
    codes, scales = mxq.quantize_cache_packed(x, fmt, B)
    wc, ws = oracle.quantize_cache_packed(bits(x), fmt, B, dtype_name)
    assert_equal(u8(codes), wc, "%s B=%d codes" % (fmt, B))
    assert_equal(u8(scales), ws, "%s B=%d scales" % (fmt, B))
    y = mxq.dequantize_cache_packed(codes, scales, fmt, B, x.dtype)
    assert_equal(bits(y), oracle.dequantize_cache_packed(wc, ws, fmt, B, x.shape[-1], dtype_name),
                 "%s B=%d unpack" % (fmt, B))
    assert_equal(bits(y), bits(mxq.quantize_cache(x, fmt, B)), "%s B=%d vs fake quant" % (fmt, B))


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("B", [8, 16, 32, 64, 128, 256])
def test_packed_fast_block_sizes(fmt, B):
    x = torch.cat([gen.kv_cache((1, 64, 512)).view(64, 512), gen.mixed_blocks(64, 512)]).to(DEV)
    check_case(x, fmt, B)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_packed_other_dtypes(fmt, dtype):
    x = torch.cat([gen.kv_cache((1, 64, 512)).view(64, 512), gen.mixed_blocks(64, 512)]).to(dtype)
    if dtype == torch.float32:
        # tiny magnitudes down to the f32 subnormals
        x.view(-1)[:4096] *= 1e-36
    x = x.to(DEV)
    for B in (16, 32, 128):
        check_case(x, fmt, B, _NAME[dtype])


@pytest.mark.parametrize("fmt,C,B", [("fp8", 120, 24), ("fp8", 33, 1), ("fp8", 21, 3),
                                     ("mxfp4", 132, 6), ("nvfp4", 40, 10), ("nvfp4", 66, 2)])
def test_packed_general_block_sizes(fmt, C, B):
    x = gen.kv_cache((1, 37, C)).view(37, C).to(DEV)
    check_case(x, fmt, B)


def test_packed_unaligned_input_takes_general_path():
    base = gen.kv_cache((1, 17, 257)).view(-1).to(DEV)
    x = torch.as_strided(base, (16, 256), (256, 1), 1)  # offset by one element
    for fmt, B in FORMATS:
        check_case(x, fmt, B)


@pytest.mark.parametrize("fmt,B", FORMATS)
def test_packed_full_kv_cache(fmt, B):
    # the bench's KV-cache tensor: the round trip against the fake
    # quantization everywhere, codes and scales against the oracle on rows
    x = gen.kv_cache(device=DEV)
    codes, scales = mxq.quantize_cache_packed(x, fmt, B)
    y = mxq.dequantize_cache_packed(codes, scales, fmt, B)
    assert torch.equal(y.view(torch.int16), mxq.quantize_cache(x, fmt, B).view(torch.int16))
    C = x.shape[-1]
    xr, cr, sr = x.view(-1, C), codes.view(-1, codes.shape[-1]), scales.view(-1, C // B)
    rows = torch.tensor([0, 1, 4095, 8191, 12345, xr.shape[0] - 1])
    wc, ws = oracle.quantize_cache_packed(bits(xr[rows.to(DEV)]), fmt, B)
    assert_equal(u8(cr[rows.to(DEV)]), wc, "sampled codes")
    assert_equal(u8(sr[rows.to(DEV)]), ws, "sampled scales")


@pytest.mark.parametrize("fmt,B", FORMATS)
def test_packed_storage_sizes(fmt, B):
    x = gen.kv_cache((2, 16, 512), device=DEV)
    codes, scales = mxq.quantize_cache_packed(x, fmt, B)
    assert codes.shape == (2, 16, 512 if fmt == "fp8" else 256)
    assert scales.shape == (2, 16, 512 // B)
    # bits per stored value: element bits plus 8 / B for the scale
    bits_per_value = 8.0 * (codes.numel() + scales.numel()) / x.numel()
    assert bits_per_value == (8 if fmt == "fp8" else 4) + 8.0 / B


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
def test_unpack_every_code_and_scale_byte(fmt):
    # every code byte against every scale byte (E8M0 0xFF and the E4M3 NaN
    # bytes included); NaN results only have to be NaN
    B = 16
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).repeat(256, 1)
    if fmt != "fp8":
        codes = codes[:, :128].contiguous()
    C = codes.shape[1] * (1 if fmt == "fp8" else 2)
    scales = torch.arange(256, dtype=torch.int32).to(torch.uint8)[:, None].repeat(1, C // B)
    for dtype in (torch.bfloat16, torch.float32):
        y = mxq.dequantize_cache_packed(codes.to(DEV), scales.to(DEV), fmt, B, dtype)
        want = oracle.dequantize_cache_packed(codes.numpy(), scales.numpy(), fmt, B, C,
                                              _NAME[dtype])
        got_nan = np.isnan(y.float().cpu().numpy())
        want_nan = np.isnan(to_float(want, dtype))
        assert np.array_equal(got_nan, want_nan), fmt
        keep = ~got_nan
        assert_equal(bits(y)[keep], want[keep], "%s %s" % (fmt, dtype))


def test_cache_quantization_function_straight_through():
    x = gen.kv_cache((2, 64, 512), device=DEV).requires_grad_(True)
    for fmt, B in FORMATS:
        y = mxq.CacheQuantization.apply(x, B, fmt)
        assert y.dtype == x.dtype and y.data_ptr() != x.data_ptr()
        assert torch.equal(y.detach().view(torch.int16),
                           mxq.quantize_cache(x.detach(), fmt, B).view(torch.int16))
        g = torch.randn_like(y)
        (gx,) = torch.autograd.grad(y, x, g)
        assert torch.equal(gx, g)
