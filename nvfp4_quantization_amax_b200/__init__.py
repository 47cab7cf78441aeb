"""Block-scaled microscaling quantization (MXFP4 / NVFP4 / FP8) on NVIDIA B200.

A thin Python binding over the C ABI of ``libmxq.so`` (declared in
``include/mxq.h``).  Each function here only checks and marshals arguments,
allocates outputs with torch and calls the library on the current CUDA
stream; every step of the computation runs in the library's sm_100a
kernels.  There is no CPU fallback: a missing library or a non-CUDA
device raises.

Inputs that live in host memory are accepted too: they are copied to the
current CUDA device (asynchronously when pinned), processed there, and the
results are copied back to host memory before the call returns.
"""
from ._abi import (  # noqa: F401
    CacheQuantization,
    MxqError,
    debug_checks,
    debug_selftest,
    lib,
    lib_path,
    mx_dequantize,
    mx_quantize,
    mxfp4_grouped_mm,
    nvfp4_dequantize,
    nvfp4_quantize,
    nvfp4_w4a4_grouped_mm,
    dequantize_cache_packed,
    quantize_cache,
    quantize_cache_packed,
    set_wait_limit_ns,
    status_string,
    w4a4_grouped_mm,
)
