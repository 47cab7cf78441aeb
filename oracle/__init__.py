"""Scalar CPU oracle for block-scaled microscaling quantization.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it; the product package never imports it.  The numeric
work happens in ``mxq_oracle.c`` (IEEE double, its own rounding routines);
this module only moves numpy arrays in and out of it.

Arrays of floating-point elements are passed as their raw bit patterns:
uint16 for bf16 / f16, uint32 for f32.
"""
import contextlib
import ctypes
import os

import numpy as np

from . import build as _build

DTYPES = {"bf16": 0, "f16": 1, "f32": 2}
FORMATS = {"fp8": 0, "mxfp4": 1, "nvfp4": 2}
_BITS = {"bf16": np.uint16, "f16": np.uint16, "f32": np.uint32}

_libs = {}
_all_cores = False

# An already-built oracle library to load instead of oracle/liboracle.so: the
# mutation tests point it at copies of the oracle with a planted mistake and
# check that the pins catch each one.
LIB_ENV = "MXQ_ORACLE_LIB"


@contextlib.contextmanager
def all_cores():
    """Within the block, calls use the OpenMP build of the same oracle
    source, whose row loops run on all host cores (identical results)."""
    global _all_cores
    prev, _all_cores = _all_cores, True
    try:
        yield
    finally:
        _all_cores = prev


def lib():
    path = os.environ.get(LIB_ENV) or _build.build(openmp=_all_cores)
    if path not in _libs:
        L = ctypes.CDLL(path)
        d, i, i64, p = ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        L.orc_e2m1_value.restype = d
        L.orc_e2m1_value.argtypes = [i]
        L.orc_e2m1_code.restype = i
        L.orc_e2m1_code.argtypes = [d]
        for name in ("orc_round_bf16", "orc_round_f16", "orc_round_f32", "orc_round_e4m3"):
            getattr(L, name).restype = d
            getattr(L, name).argtypes = [d]
        L.orc_encode_e4m3.restype = ctypes.c_uint8
        L.orc_encode_e4m3.argtypes = [d]
        L.orc_decode_e4m3.restype = d
        L.orc_decode_e4m3.argtypes = [ctypes.c_uint8]
        L.orc_decode_array.argtypes = [p, i, i64, p]
        L.orc_round_array.argtypes = [p, i, i64, p]
        L.orc_mx_scale_exp.restype = i
        L.orc_mx_scale_exp.argtypes = [d]
        L.orc_mx_quantize.restype = i
        L.orc_mx_quantize.argtypes = [p, i, i64, i64, p, p]
        L.orc_mx_dequantize.restype = i
        L.orc_mx_dequantize.argtypes = [p, p, i64, i64, p, i]
        L.orc_cache_scale_exp.restype = i
        L.orc_cache_scale_exp.argtypes = [d, i]
        L.orc_cache_element.restype = d
        L.orc_cache_element.argtypes = [d, i, i]
        L.orc_quantize_cache.restype = i
        L.orc_quantize_cache.argtypes = [p, p, i, i64, i64, i, i]
        L.orc_check_offs.restype = i
        L.orc_check_offs.argtypes = [p, i64, i64]
        L.orc_nvfp4_global_scale.restype = d
        L.orc_nvfp4_global_scale.argtypes = [d]
        L.orc_nvfp4_block_scale.restype = d
        L.orc_nvfp4_block_scale.argtypes = [d, d]
        L.orc_nvfp4_quantize.restype = i
        L.orc_nvfp4_quantize.argtypes = [p, i, i64, i64, p, p, p]
        L.orc_nvfp4_block_sq_error.restype = d
        L.orc_nvfp4_block_sq_error.argtypes = [p, d, i]
        L.orc_nvfp4_mse_code.restype = i
        L.orc_nvfp4_mse_code.argtypes = [p, d]
        L.orc_nvfp4_quantize_mse_rows.restype = i
        L.orc_nvfp4_quantize_mse_rows.argtypes = [p, i, i64, i64, d, p, p]
        L.orc_nvfp4_quantize_mse.restype = i
        L.orc_nvfp4_quantize_mse.argtypes = [p, i, i64, i64, p, p, p]
        L.orc_nvfp4_dequantize.restype = i
        L.orc_nvfp4_dequantize.argtypes = [p, p, ctypes.c_float, i64, i64, p, i]
        L.orc_cache_scale_byte.restype = ctypes.c_uint8
        L.orc_cache_scale_byte.argtypes = [i, i]
        L.orc_quantize_cache_packed.restype = i
        L.orc_quantize_cache_packed.argtypes = [p, i, i64, i64, i, i, p, p]
        L.orc_dequantize_cache_packed.restype = i
        L.orc_dequantize_cache_packed.argtypes = [p, p, i64, i64, i, i, p, i]
        L.orc_w4a4_grouped_mm.restype = i
        L.orc_w4a4_grouped_mm.argtypes = [p, p, p, p, i64, i64, i64, i64, p, i64, p]
        L.orc_nvfp4_quantize_rows.restype = i
        L.orc_nvfp4_quantize_rows.argtypes = [p, i, i64, i64, d, p, p]
        L.orc_nvfp4_w4a4_grouped_mm.restype = i
        L.orc_nvfp4_w4a4_grouped_mm.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, i64, p]
        L.orc_grouped_mm.restype = i
        L.orc_grouped_mm.argtypes = [p, p, p, p, i64, i64, i64, i64, i, p, i64, p]
        _libs[path] = L
    return _libs[path]


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- scalar helpers -------------------------------------------------------

def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e2m1_code(v):
    return lib().orc_e2m1_code(float(v))


def round_bf16(v):
    return lib().orc_round_bf16(float(v))


def round_f16(v):
    return lib().orc_round_f16(float(v))


def round_f32(v):
    return lib().orc_round_f32(float(v))


def round_e4m3(v):
    return lib().orc_round_e4m3(float(v))


def encode_e4m3(v):
    return lib().orc_encode_e4m3(float(v))


def decode_e4m3(b):
    return lib().orc_decode_e4m3(int(b))


def mx_scale_exp(amax):
    return lib().orc_mx_scale_exp(float(amax))


def cache_scale_exp(amax, fmt):
    return lib().orc_cache_scale_exp(float(amax), FORMATS[fmt])


def cache_element(x, k, fmt):
    return lib().orc_cache_element(float(x), int(k), FORMATS[fmt])


# ---- array helpers --------------------------------------------------------

def decode(bits, dtype):
    """Bit patterns of `dtype` -> float64 values."""
    b = _c(bits, _BITS[dtype])
    out = np.empty(b.shape, np.float64)
    lib().orc_decode_array(_ptr(b), DTYPES[dtype], b.size, _ptr(out))
    return out


def round_to(values, dtype):
    """float64 values -> bit patterns of `dtype` (nearest-even)."""
    v = _c(values, np.float64)
    out = np.empty(v.shape, _BITS[dtype])
    lib().orc_round_array(_ptr(v), DTYPES[dtype], v.size, _ptr(out))
    return out


def mx_quantize(x_bits, dtype="bf16"):
    """x [..., K] -> (packed uint8 [..., K/2], scales uint8 [..., K/32])."""
    x = _c(x_bits, _BITS[dtype])
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.empty(x.shape[:-1] + (K // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (K // 32,), np.uint8)
    rc = lib().orc_mx_quantize(_ptr(x), DTYPES[dtype], rows, K, _ptr(packed), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle mx_quantize: bad arguments (K %% 32 != 0?) rc=%d" % rc)
    return packed, scales


def mx_dequantize(packed, scales, dtype="bf16"):
    """packed [..., K/2], scales [..., K/32] -> bits of dtype [..., K]."""
    p = _c(packed, np.uint8)
    s = _c(scales, np.uint8)
    K = p.shape[-1] * 2
    rows = p.size // p.shape[-1] if p.shape[-1] else 0
    out = np.empty(p.shape[:-1] + (K,), _BITS[dtype])
    rc = lib().orc_mx_dequantize(_ptr(p), _ptr(s), rows, K, _ptr(out), DTYPES[dtype])
    if rc != 0:
        raise ValueError("oracle mx_dequantize: bad arguments rc=%d" % rc)
    return out


def quantize_cache(x_bits, fmt, block_size, dtype="bf16"):
    """Fake quantization of x [..., C]; returns bits of the same dtype."""
    x = _c(x_bits, _BITS[dtype])
    C = x.shape[-1]
    rows = x.size // C if C else 0
    out = np.empty_like(x)
    rc = lib().orc_quantize_cache(_ptr(x), _ptr(out), DTYPES[dtype], rows, C, FORMATS[fmt],
                                  int(block_size))
    if rc != 0:
        raise ValueError("oracle quantize_cache: bad arguments rc=%d" % rc)
    return out


def check_offs(offs, T):
    o = _c(offs, np.int32)
    return lib().orc_check_offs(_ptr(o), o.size, int(T)) == 0


def grouped_mm(a_bits, packed, scales, offs, transpose_w=False, rows=None):
    """Exact-sum (double) grouped GEMM on the listed rows (default: all).

    a_bits: bf16 bits [T, Kin]; packed [E, N, K/2]; scales [E, N, K/32];
    offs int32 [E] (inclusive prefix sums of the expert row counts).
    Returns float64 [len(rows), Nout], not rounded.
    """
    a = _c(a_bits, np.uint16)
    p = _c(packed, np.uint8)
    s = _c(scales, np.uint8)
    o = _c(offs, np.int32)
    E, N, Kh = p.shape
    K = 2 * Kh
    T = a.shape[0]
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    r = _c(rows, np.int64)
    nout = K if transpose_w else N
    out = np.zeros((r.size, nout), np.float64)
    rc = lib().orc_grouped_mm(_ptr(a), _ptr(p), _ptr(s), _ptr(o), T, E, N, K,
                              1 if transpose_w else 0, _ptr(r), r.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle grouped_mm: rc=%d" % rc)
    return out



def w4a4_grouped_mm(x_bits, packed, scales, offs, rows=None):
    """Exact-sum grouped GEMM with the activations quantized to MXFP4 first:
    out[i, n] = sum_k deq(mx_quantize(x))[t, k] W_e[n, k], t = rows[i]."""
    x = _c(x_bits, np.uint16)
    p = _c(packed, np.uint8)
    s = _c(scales, np.uint8)
    o = _c(offs, np.int32)
    E, N, Kh = p.shape
    K = 2 * Kh
    T = x.shape[0]
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    r = _c(rows, np.int64)
    out = np.zeros((r.size, N), np.float64)
    rc = lib().orc_w4a4_grouped_mm(_ptr(x), _ptr(p), _ptr(s), _ptr(o), T, E, N, K, _ptr(r),
                                   r.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle w4a4_grouped_mm: rc=%d" % rc)
    return out


def nvfp4_global_scale(amax):
    return lib().orc_nvfp4_global_scale(float(amax))


def nvfp4_block_scale(amax_b, g):
    return lib().orc_nvfp4_block_scale(float(amax_b), float(g))


def nvfp4_quantize(x_bits, dtype="bf16"):
    """x [..., K] (K % 16 == 0) -> (packed uint8 [..., K/2], E4M3 block scales
    uint8 [..., K/16], global scale g as a Python float)."""
    x = _c(x_bits, _BITS[dtype])
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.empty(x.shape[:-1] + (K // 2,), np.uint8)
    bs = np.empty(x.shape[:-1] + (K // 16,), np.uint8)
    g = ctypes.c_float(0.0)
    rc = lib().orc_nvfp4_quantize(_ptr(x), DTYPES[dtype], rows, K, _ptr(packed), _ptr(bs),
                                  ctypes.byref(g))
    if rc != 0:
        raise ValueError("oracle nvfp4_quantize: bad arguments rc=%d" % rc)
    return packed, bs, g.value


def nvfp4_dequantize(packed, block_scales, global_scale, dtype="bf16"):
    p = _c(packed, np.uint8)
    s = _c(block_scales, np.uint8)
    K = p.shape[-1] * 2
    rows = p.size // p.shape[-1] if p.shape[-1] else 0
    out = np.empty(p.shape[:-1] + (K,), _BITS[dtype])
    rc = lib().orc_nvfp4_dequantize(_ptr(p), _ptr(s), float(global_scale), rows, K, _ptr(out),
                                    DTYPES[dtype])
    if rc != 0:
        raise ValueError("oracle nvfp4_dequantize: bad arguments rc=%d" % rc)
    return out


def quantize_cache_packed(x_bits, fmt, block_size, dtype="bf16"):
    """Stored form of quantize_cache: (codes, scale bytes)."""
    x = _c(x_bits, _BITS[dtype])
    C = x.shape[-1]
    rows = x.size // C if C else 0
    ncode = C if fmt == "fp8" else C // 2
    codes = np.zeros(x.shape[:-1] + (ncode,), np.uint8)
    scales = np.empty(x.shape[:-1] + (C // int(block_size),), np.uint8)
    rc = lib().orc_quantize_cache_packed(_ptr(x), DTYPES[dtype], rows, C, FORMATS[fmt],
                                         int(block_size), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle quantize_cache_packed: bad arguments rc=%d" % rc)
    return codes, scales


def dequantize_cache_packed(codes, scales, fmt, block_size, channels, dtype="bf16"):
    c = _c(codes, np.uint8)
    s = _c(scales, np.uint8)
    C = int(channels)
    rows = s.size // (C // int(block_size))
    out = np.empty(s.shape[:-1] + (C,), _BITS[dtype])
    rc = lib().orc_dequantize_cache_packed(_ptr(c), _ptr(s), rows, C, FORMATS[fmt],
                                           int(block_size), _ptr(out), DTYPES[dtype])
    if rc != 0:
        raise ValueError("oracle dequantize_cache_packed: bad arguments rc=%d" % rc)
    return out


def cache_scale_byte(k, fmt):
    return lib().orc_cache_scale_byte(int(k), FORMATS[fmt])


def nvfp4_block_sq_error(w16, g, code):
    """Squared weight error of one 16-block (float64 values) under an E4M3
    block-scale code."""
    w = np.ascontiguousarray(w16, np.float64)
    assert w.size == 16
    return lib().orc_nvfp4_block_sq_error(_ptr(w), float(g), int(code))


def nvfp4_mse_code(w16, g):
    w = np.ascontiguousarray(w16, np.float64)
    assert w.size == 16
    return lib().orc_nvfp4_mse_code(_ptr(w), float(g))


def nvfp4_quantize_mse(x_bits, dtype="bf16", g=None):
    """NVFP4 with mse block scales -> (packed, block scales, g).  With g
    given, rows are quantized with that per-tensor scale (for samples of a
    larger tensor)."""
    x = _c(x_bits, _BITS[dtype])
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.empty(x.shape[:-1] + (K // 2,), np.uint8)
    bs = np.empty(x.shape[:-1] + (K // 16,), np.uint8)
    if g is None:
        gf = ctypes.c_float(0.0)
        rc = lib().orc_nvfp4_quantize_mse(_ptr(x), DTYPES[dtype], rows, K, _ptr(packed),
                                          _ptr(bs), ctypes.byref(gf))
        g = gf.value
    else:
        rc = lib().orc_nvfp4_quantize_mse_rows(_ptr(x), DTYPES[dtype], rows, K, float(g),
                                               _ptr(packed), _ptr(bs))
    if rc != 0:
        raise ValueError("oracle nvfp4_quantize_mse: bad arguments rc=%d" % rc)
    return packed, bs, g


def nvfp4_quantize_rows(x_bits, g, dtype="bf16"):
    """NVFP4 codes and block scales of rows with a given per-tensor scale g."""
    x = _c(x_bits, _BITS[dtype])
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.empty(x.shape[:-1] + (K // 2,), np.uint8)
    bs = np.empty(x.shape[:-1] + (K // 16,), np.uint8)
    rc = lib().orc_nvfp4_quantize_rows(_ptr(x), DTYPES[dtype], rows, K, float(g), _ptr(packed),
                                       _ptr(bs))
    if rc != 0:
        raise ValueError("oracle nvfp4_quantize_rows: bad arguments rc=%d" % rc)
    return packed, bs


def nvfp4_w4a4_grouped_mm(x_bits, packed, block_scales, w_global, offs, rows=None):
    """Exact-sum grouped GEMM of NVFP4 activations (x quantized as one
    tensor) with NVFP4 expert weights (one global scale per expert)."""
    x = _c(x_bits, np.uint16)
    p = _c(packed, np.uint8)
    s = _c(block_scales, np.uint8)
    gw = _c(w_global, np.float32)
    o = _c(offs, np.int32)
    E, N, Kh = p.shape
    K = 2 * Kh
    T = x.shape[0]
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    r = _c(rows, np.int64)
    out = np.zeros((r.size, N), np.float64)
    rc = lib().orc_nvfp4_w4a4_grouped_mm(_ptr(x), _ptr(p), _ptr(s), _ptr(gw), _ptr(o), T, E, N, K,
                                         _ptr(r), r.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle nvfp4_w4a4_grouped_mm: rc=%d" % rc)
    return out
