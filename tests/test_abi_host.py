"""Host-side checks of the C ABI: the library loads, exports every function
include/mxq.h declares, and rejects bad arguments before launching anything
(every call here fails validation or is a no-op, so no GPU is touched)."""
import ctypes
import os
import re
import subprocess

import pytest

import nvfp4_quantization_amax_b200 as mxq
from nvfp4_quantization_amax_b200 import build as mxq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")

OK, EARG, ESHAPE, EALIGN, EUNSUP = 0, -1, -2, -3, -4
NULL = None
BAD = ctypes.c_void_p(0x1001)  # misaligned, never dereferenced
A1, A2 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)  # never dereferenced


@pytest.fixture(scope="module")
def L():
    mxq_build.build()
    return mxq.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^(?:int|uint64_t|const char\*)\s+(\w+)\(", text, re.M)


def test_header_declares_the_boundary():
    assert set(declared_functions()) >= {"mx_quantize", "mx_dequantize", "quantize_cache",
                                         "mxfp4_grouped_mm", "mxq_status_string", "mxq_version",
                                         "mxq_set_wait_limit_ns"}


def test_library_exports_every_declared_symbol(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", mxq.lib_path()]).decode()
    exported = set(re.findall(r"\sT\s(\w+)$", out, re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_library_is_built_for_sm100a_only():
    assert mxq_build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "--use_fast_math" not in mxq_build.FLAGS and "-lineinfo" in mxq_build.FLAGS


def test_status_strings(L):
    assert mxq.status_string(0) == "MXQ_OK"
    assert mxq.status_string(-6) == "MXQ_ERR_BAD_OFFS"
    assert mxq.status_string(-7) == "MXQ_ERR_TIMEOUT"
    assert mxq.status_string(-99) == "MXQ_ERR_UNKNOWN"
    assert L.mxq_version() >= 100


def test_mx_quantize_validation(L):
    assert L.mx_quantize(NULL, 0, 4, 64, NULL, NULL, NULL) == EARG
    assert L.mx_quantize(A1, 0, 4, 48, A2, A2, NULL) == ESHAPE
    assert L.mx_quantize(A1, 0, -1, 64, A2, A2, NULL) == ESHAPE
    assert L.mx_quantize(A1, 7, 4, 64, A2, A2, NULL) == EARG
    assert L.mx_quantize(BAD, 0, 4, 64, A2, A2, NULL) == EALIGN
    assert L.mx_quantize(A1, 0, 4, 64, BAD, A2, NULL) == EALIGN
    assert L.mx_quantize(NULL, 0, 0, 64, NULL, NULL, NULL) == OK  # empty: no-op


def test_mx_dequantize_validation(L):
    assert L.mx_dequantize(NULL, NULL, 4, 64, NULL, 0, NULL) == EARG
    assert L.mx_dequantize(A1, A2, 4, 40, A1, 0, NULL) == ESHAPE
    assert L.mx_dequantize(A1, A2, 4, 64, A1, 3, NULL) == EARG
    assert L.mx_dequantize(BAD, A2, 4, 64, A1, 0, NULL) == EALIGN
    assert L.mx_dequantize(A1, A2, 4, 64, BAD, 0, NULL) == EALIGN
    assert L.mx_dequantize(NULL, NULL, 4, 0, NULL, 0, NULL) == OK


def test_quantize_cache_validation(L):
    assert L.quantize_cache(NULL, NULL, 0, 4, 64, 0, 32, NULL) == EARG
    assert L.quantize_cache(A1, A2, 0, 4, 64, 5, 32, NULL) == EARG
    assert L.quantize_cache(A1, A2, 9, 4, 64, 0, 32, NULL) == EARG
    assert L.quantize_cache(A1, A2, 0, 4, 64, 0, 0, NULL) == ESHAPE
    assert L.quantize_cache(A1, A2, 0, -4, 64, 0, 16, NULL) == ESHAPE
    # the output must be independent storage: overlapping in/out is rejected
    assert L.quantize_cache(A1, A1, 0, 4, 64, 0, 16, NULL) == EARG
    assert L.quantize_cache(A1, ctypes.c_void_p(0x10000 + 64), 0, 4, 64, 1, 32, NULL) == EARG
    assert L.quantize_cache(NULL, NULL, 0, 0, 64, 0, 16, NULL) == OK


def test_grouped_mm_validation(L):
    f = L.mxfp4_grouped_mm
    assert f(A1, A2, A2, A2, 8, 0, 16, 64, 0, A1, NULL, NULL) == ESHAPE  # E < 1
    assert f(A1, A2, A2, A2, 8, 2, 16, 48, 0, A1, NULL, NULL) == ESHAPE  # K % 32
    assert f(A1, A2, A2, A2, 8, 2, 0, 64, 0, A1, NULL, NULL) == ESHAPE  # N < 1
    assert f(A1, A2, A2, A2, -1, 2, 16, 64, 0, A1, NULL, NULL) == ESHAPE
    assert f(A1, A2, A2, A2, 8, 2, 16, 64, 2, A1, NULL, NULL) == EARG  # transpose flag
    assert f(A1, A2, A2, NULL, 8, 2, 16, 64, 0, A1, NULL, NULL) == EARG  # offs
    assert f(NULL, A2, A2, A2, 8, 2, 16, 64, 0, A1, NULL, NULL) == EARG  # a
    assert f(A1, A2, A2, A2, 0, 2, 16, 64, 0, A1, NULL, NULL) == OK  # T == 0: no-op
    # bf16 a / y off their 2-byte boundary, int32 offs / status off 4 bytes:
    # rejected on the host (the general kernel would fault on them)
    Y, OFFS = ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000)
    assert f(BAD, A2, A2, OFFS, 8, 2, 16, 64, 0, Y, NULL, NULL) == EALIGN
    assert f(A1, A2, A2, OFFS, 8, 2, 16, 64, 1, BAD, NULL, NULL) == EALIGN
    assert f(A1, A2, A2, ctypes.c_void_p(0x50002), 8, 2, 16, 64, 0, Y, NULL, NULL) == EALIGN
    assert f(A1, A2, A2, OFFS, 8, 2, 16, 64, 0, Y, ctypes.c_void_p(0x60002), NULL) == EALIGN


def test_binding_fails_loudly_without_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    with pytest.raises(RuntimeError):
        mxq.quantize_cache(torch.zeros(4, 32, dtype=torch.bfloat16), "fp8", 32)


def test_debug_entry_points_are_unsupported_in_the_normal_library(L):
    rec = (ctypes.c_int64 * 3)(7, 7, 7)
    assert L.mxq_debug_checks(ctypes.cast(rec, ctypes.c_void_p)) == EUNSUP
    assert list(rec) == [0, 0, 0]
    assert L.mxq_debug_checks(NULL) == EARG
    assert L.mxq_debug_selftest(A1, NULL) == EUNSUP  # nothing launched
    assert L.mxq_debug_selftest(BAD, NULL) == EALIGN


def test_wait_limit_setter_round_trips(L):
    prev = mxq.set_wait_limit_ns(123)
    assert mxq.set_wait_limit_ns(prev) == 123


def test_nvfp4_validation(L):
    assert L.nvfp4_quantize(A1, 0, 4, 40, A2, A2, A2, A1, NULL) == ESHAPE
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, A2, A2, NULL, NULL) == EARG  # workspace
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, A2, NULL, A1, NULL) == EARG  # global scale
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, A2, A2, BAD, NULL) == EALIGN
    assert L.nvfp4_quantize(BAD, 0, 4, 64, A2, A2, A2, A1, NULL) == EALIGN
    # the global scale is one float the kernels read or write: 4-byte aligned
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, A2, BAD, A1, NULL) == EALIGN
    assert L.nvfp4_quantize(NULL, 0, 0, 64, NULL, NULL, BAD, A1, NULL) == EALIGN
    assert L.nvfp4_quantize_mse(A1, 0, 4, 64, A2, A2, BAD, A1, NULL) == EALIGN
    assert L.nvfp4_quantize(A1, 9, 4, 64, A2, A2, A2, A1, NULL) == EARG
    assert L.nvfp4_dequantize(A1, A2, A2, 4, 24, A1, 0, NULL) == ESHAPE
    assert L.nvfp4_dequantize(A1, A2, NULL, 4, 32, A1, 0, NULL) == EARG
    assert L.nvfp4_dequantize(BAD, A2, A2, 4, 32, A1, 0, NULL) == EALIGN
    assert L.nvfp4_dequantize(A1, A2, BAD, 4, 32, A1, 0, NULL) == EALIGN
    assert L.nvfp4_dequantize(NULL, NULL, NULL, 0, 32, NULL, 0, NULL) == OK


def test_nvfp4_noalloc_validation_needs_no_gpu(L):
    # argument errors are reported before the scratch is looked up
    assert L.nvfp4_quantize_noalloc(A1, 0, 4, 40, A2, A2, A2, NULL) == ESHAPE
    assert L.nvfp4_quantize_noalloc(A1, 0, 4, 64, A2, A2, NULL, NULL) == EARG
    assert L.nvfp4_quantize_noalloc(BAD, 0, 4, 64, A2, A2, A2, NULL) == EALIGN
    assert L.nvfp4_quantize_noalloc(A1, 0, 4, 64, A2, A2, BAD, NULL) == EALIGN
    assert L.nvfp4_quantize_noalloc(A1, 5, 4, 64, A2, A2, A2, NULL) == EARG


def test_packed_cache_validation(L):
    q, d = L.quantize_cache_packed, L.dequantize_cache_packed
    assert q(A1, 0, 4, 64, 3, 32, A2, A2, NULL) == EARG  # format
    assert q(A1, 7, 4, 64, 0, 32, A2, A2, NULL) == EARG  # dtype
    assert q(A1, 0, 4, 64, 0, 0, A2, A2, NULL) == ESHAPE  # block_size < 1
    assert q(A1, 0, 4, 60, 0, 32, A2, A2, NULL) == ESHAPE  # no partial group is stored
    assert q(A1, 0, 4, 63, 1, 21, A2, A2, NULL) == ESHAPE  # odd fp4 block
    assert q(A1, 0, -1, 64, 0, 32, A2, A2, NULL) == ESHAPE
    assert q(A1, 0, 4, 64, 0, 32, NULL, A2, NULL) == EARG
    assert q(BAD, 0, 4, 64, 0, 32, A2, A2, NULL) == EALIGN  # element alignment
    assert q(NULL, 0, 0, 64, 0, 32, NULL, NULL, NULL) == OK  # rows == 0: no-op
    assert d(A1, A2, 4, 64, 2, 16, BAD, 0, NULL) == EALIGN
    assert d(A1, A2, 4, 64, 2, 15, A1, 0, NULL) == ESHAPE
    assert d(A1, NULL, 4, 64, 2, 16, A1, 0, NULL) == EARG
    assert d(NULL, NULL, 4, 0, 2, 16, NULL, 0, NULL) == OK


def test_cache_quantization_function_passes_the_gradient_through():
    # backward alone needs no GPU: the straight-through gradient is returned
    # unchanged with no gradients for block_size and format
    import torch
    g = torch.randn(3, 64)
    out = mxq.CacheQuantization.backward(None, g)
    assert out[0] is g and out[1] is None and out[2] is None


def test_nvfp4_mse_validation(L):
    f = L.nvfp4_quantize_mse
    assert f(A1, 0, 4, 40, A2, A2, A2, A1, NULL) == ESHAPE
    assert f(A1, 0, 4, 64, A2, A2, A2, NULL, NULL) == EARG  # workspace
    assert f(A1, 0, 4, 64, A2, A2, NULL, A1, NULL) == EARG  # global scale
    assert f(BAD, 0, 4, 64, A2, A2, A2, A1, NULL) == EALIGN
    assert f(A1, 3, 4, 64, A2, A2, A2, A1, NULL) == EARG
    with pytest.raises(ValueError):
        import torch
        mxq.nvfp4_quantize(torch.zeros(2, 16, dtype=torch.bfloat16), rule="least")


def test_w4a4_validation(L):
    f = L.mxfp4_w4a4_grouped_mm
    assert f(A1, A1, A2, A2, A2, 8, 0, 128, 256, A1, NULL, NULL) == ESHAPE  # E < 1
    assert f(A1, A1, A2, A2, A2, 8, 2, 128, 48, A1, NULL, NULL) == ESHAPE  # K % 32
    assert f(A1, A1, A2, A2, NULL, 8, 2, 128, 256, A1, NULL, NULL) == EARG  # offs
    assert f(A1, A1, A2, A2, A2, 8, 2, 128, 96, A1, NULL, NULL) == EUNSUP  # K % 256
    assert f(A1, A1, A2, A2, A2, 8, 2, 64, 256, A1, NULL, NULL) == EUNSUP  # N % 128
    assert f(BAD, A1, A2, A2, A2, 8, 2, 128, 256, A1, NULL, NULL) == EALIGN
    assert f(A1, A1, A2, A2, ctypes.c_void_p(0x20002), 8, 2, 128, 256, A1, NULL, NULL) == EALIGN
    assert f(A1, A1, A2, A2, A2, 8, 2, 128, 256, A1, ctypes.c_void_p(0x60001), NULL) == EALIGN
    assert f(A1, A1, A2, A2, A2, 0, 2, 128, 256, A1, NULL, NULL) == OK  # T == 0


def test_nvfp4_w4a4_validation(L):
    f = L.nvfp4_w4a4_grouped_mm
    assert f(A1, A1, A2, A2, A2, A2, A2, 8, 0, 128, 256, A1, NULL, NULL) == ESHAPE  # E < 1
    assert f(A1, A1, A2, A2, A2, A2, A2, 8, 2, 128, 40, A1, NULL, NULL) == ESHAPE  # K % 16
    assert f(A1, A1, A2, A2, A2, NULL, A2, 8, 2, 128, 256, A1, NULL, NULL) == EARG  # w scales
    assert f(A1, A1, NULL, A2, A2, A2, A2, 8, 2, 128, 256, A1, NULL, NULL) == EARG  # x scale
    assert f(A1, A1, A2, A2, A2, A2, A2, 8, 2, 128, 96, A1, NULL, NULL) == EUNSUP
    assert f(BAD, A1, A2, A2, A2, A2, A2, 8, 2, 128, 256, A1, NULL, NULL) == EALIGN
    assert f(A1, A1, ctypes.c_void_p(0x20001), A2, A2, A2, A2, 8, 2, 128, 256, A1, NULL,
             NULL) == EALIGN  # x global scale
    assert f(A1, A1, A2, A2, A2, A2, ctypes.c_void_p(0x20006), 8, 2, 128, 256, A1, NULL,
             NULL) == EALIGN  # offs
    assert f(A1, A1, A2, A2, A2, A2, A2, 0, 2, 128, 256, A1, NULL, NULL) == OK


A3 = ctypes.c_void_p(0x30000)  # never dereferenced
BIG = 1 << 40


def test_outputs_that_alias_are_rejected(L):
    # x [4, 64] bf16 at A1 (512 bytes): packed inside it
    assert L.mx_quantize(A1, 0, 4, 64, ctypes.c_void_p(0x10100), A2, NULL) == EARG
    assert L.mx_quantize(A1, 0, 4, 64, A2, ctypes.c_void_p(0x20010), NULL) == EARG  # scales in packed
    assert L.mx_dequantize(A1, A2, 4, 64, A1, 0, NULL) == EARG  # out over packed
    assert L.mx_dequantize(A1, A2, 4, 64, ctypes.c_void_p(0x1FF00), 0, NULL) == EARG  # out reaches scales
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, A2, A3, ctypes.c_void_p(0x30010), NULL) == EARG
    assert L.nvfp4_quantize(A1, 0, 4, 64, A2, ctypes.c_void_p(0x20080), A1, A3, NULL) == EARG
    assert L.nvfp4_quantize_mse(A1, 0, 4, 64, A2, A2, A3, ctypes.c_void_p(0x30010), NULL) == EARG
    assert L.nvfp4_quantize_noalloc(A1, 0, 4, 64, A2, ctypes.c_void_p(0x20010), A3, NULL) == EARG
    assert L.nvfp4_dequantize(A1, A2, A3, 4, 64, ctypes.c_void_p(0x1FF80), 0, NULL) == EARG
    q, d = L.quantize_cache_packed, L.dequantize_cache_packed
    assert q(A1, 0, 4, 64, 0, 32, A1, A2, NULL) == EARG  # codes over the input
    assert q(A1, 0, 4, 64, 1, 32, A2, ctypes.c_void_p(0x20020), NULL) == EARG  # scales in codes
    assert d(A1, A2, 4, 64, 2, 16, ctypes.c_void_p(0x1FFF0), 0, NULL) == EARG
    # grouped GEMMs: y over the activations, or the status word inside y
    assert L.mxfp4_grouped_mm(A1, A2, A3, A3, 8, 2, 128, 256, 0, A1, NULL, NULL) == EARG
    assert L.mxfp4_grouped_mm(A1, A2, A3, A3, 8, 2, 128, 256, 0, ctypes.c_void_p(0x40000),
                              ctypes.c_void_p(0x40010), NULL) == EARG
    assert L.mxfp4_w4a4_grouped_mm(A1, A1, A2, A2, A3, 8, 2, 128, 256, A1, NULL, NULL) == EARG
    assert L.nvfp4_w4a4_grouped_mm(A1, A1, A1, A2, A2, A2, A3, 8, 2, 128, 256, A3, NULL,
                                   NULL) == EARG


def test_sizes_beyond_62_bits_are_rejected(L):
    assert L.mx_quantize(A1, 0, BIG, BIG, A2, A3, NULL) == ESHAPE
    assert L.mx_dequantize(A1, A2, BIG, BIG, A3, 0, NULL) == ESHAPE
    assert L.quantize_cache(A1, A2, 0, BIG, BIG, 0, 32, NULL) == ESHAPE
    assert L.nvfp4_quantize(A1, 0, BIG, BIG, A2, A2, A3, A3, NULL) == ESHAPE
    assert L.nvfp4_dequantize(A1, A2, A3, BIG, BIG, A3, 0, NULL) == ESHAPE
    assert L.quantize_cache_packed(A1, 0, BIG, 1 << 30, 0, 32, A2, A3, NULL) == ESHAPE
    assert L.mxfp4_grouped_mm(A1, A2, A3, A3, BIG, 2, 128, BIG, 0, A1, NULL, NULL) == ESHAPE


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "mxq.h"

int main(void) {
  char buf[64];
  int64_t x[8];
  /* argument errors come back before anything touches a GPU */
  int a = mx_quantize(NULL, MXQ_BF16, 4, 64, NULL, NULL, NULL);
  int b = mx_quantize(x, MXQ_BF16, 4, 48, x, x, NULL);
  int c = quantize_cache(x, x, MXQ_BF16, 1, 8, MXQ_FMT_NVFP4, 16, NULL);
  int d = nvfp4_quantize(x, MXQ_F32, 2, 40, x, x, (float*)x, x, NULL);
  int e = mxfp4_grouped_mm(x, x, x, (const int32_t*)x, 8, 0, 128, 256, 0, x, NULL, NULL);
  snprintf(buf, sizeof buf, "%s", mxq_status_string(a));
  printf("%d %d %d %d %d %s %d %d\n", a, b, c, d, e, buf, mxq_version() >= 100,
         MXQ_NVFP4_WORKSPACE_BYTES);
  return strcmp(buf, "MXQ_ERR_INVALID_ARG") != 0;
}
"""


def test_plain_c_program_builds_against_the_header_and_links(tmp_path, L):
    # the boundary is a C ABI: a C11 program (no C++, no CUDA headers) that
    # includes include/mxq.h and links libmxq.so sees every status above
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(mxq._abi.lib_path())
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                           os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lmxq",
                           "-Wl,-rpath," + libdir, "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == [str(EARG), str(ESHAPE), str(EARG), str(ESHAPE), str(ESHAPE),
                                  "MXQ_ERR_INVALID_ARG", "1", "16"]
    # the same program as C++ (the header's extern "C" block) links the same symbols
    exe_cc = tmp_path / "consumer_cc"
    subprocess.check_call(["g++", "-x", "c++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I",
                           os.path.join(ROOT, "include"), str(src), "-x", "none", "-L", libdir,
                           "-lmxq", "-Wl,-rpath," + libdir, "-o", str(exe_cc)])
    out_cc = subprocess.run([str(exe_cc)], capture_output=True, text=True, timeout=60)
    assert out_cc.returncode == 0 and out_cc.stdout == out.stdout


def _base(i):
    # distinct, widely spaced stand-in device addresses (never dereferenced)
    return (i + 1) << 24


# Every pointer the header documents as aligned: (entry point, argument
# template with ("P", i) for the i-th stand-in pointer, {argument index:
# the boundary it must sit on}).  Sizes are small and valid, so each call
# below fails only on the one pointer moved off its boundary.
_ALIGNED_POINTERS = [
    ("mx_quantize", [("P", 0), 0, 4, 64, ("P", 1), ("P", 2), NULL], {0: 16, 4: 16}),
    ("mx_dequantize", [("P", 0), ("P", 1), 4, 64, ("P", 2), 0, NULL], {0: 16, 4: 16}),
    ("quantize_cache", [("P", 0), ("P", 1), 0, 4, 64, 0, 32, NULL], {0: 2, 1: 2}),
    ("quantize_cache", [("P", 0), ("P", 1), 2, 4, 64, 1, 32, NULL], {0: 4, 1: 4}),
    ("quantize_cache_packed", [("P", 0), 0, 4, 64, 1, 32, ("P", 1), ("P", 2), NULL], {0: 2}),
    ("dequantize_cache_packed", [("P", 0), ("P", 1), 4, 64, 1, 32, ("P", 2), 0, NULL], {6: 2}),
    ("mxfp4_grouped_mm",
     [("P", 0), ("P", 1), ("P", 2), ("P", 3), 8, 1, 128, 256, 0, ("P", 4), ("P", 5), NULL],
     {0: 2, 3: 4, 9: 2, 10: 4}),
    ("mxfp4_w4a4_grouped_mm",
     [("P", 0), ("P", 1), ("P", 2), ("P", 3), ("P", 4), 8, 1, 128, 256, ("P", 5), ("P", 6), NULL],
     {0: 16, 1: 16, 2: 16, 3: 16, 4: 4, 9: 16, 10: 4}),
    ("nvfp4_w4a4_grouped_mm",
     [("P", 0), ("P", 1), ("P", 2), ("P", 3), ("P", 4), ("P", 5), ("P", 6), 8, 1, 128, 256,
      ("P", 7), ("P", 8), NULL],
     {0: 16, 1: 16, 2: 4, 3: 16, 4: 16, 5: 4, 6: 4, 11: 16, 12: 4}),
    ("nvfp4_quantize", [("P", 0), 0, 4, 64, ("P", 1), ("P", 2), ("P", 3), ("P", 4), NULL],
     {0: 16, 4: 16, 6: 4, 7: 16}),
    ("nvfp4_quantize_mse", [("P", 0), 0, 4, 64, ("P", 1), ("P", 2), ("P", 3), ("P", 4), NULL],
     {0: 16, 4: 16, 6: 4, 7: 16}),
    ("nvfp4_quantize_noalloc", [("P", 0), 0, 4, 64, ("P", 1), ("P", 2), ("P", 3), NULL],
     {0: 16, 4: 16, 6: 4}),
    ("nvfp4_dequantize", [("P", 0), ("P", 1), ("P", 2), 4, 64, ("P", 3), 0, NULL],
     {0: 16, 2: 4, 5: 16}),
    ("mxq_debug_selftest", [("P", 0), NULL], {0: 4}),
]


@pytest.mark.parametrize("name,template,rules", _ALIGNED_POINTERS,
                         ids=["%s-%d" % (e[0], i) for i, e in enumerate(_ALIGNED_POINTERS)])
def test_every_aligned_pointer_is_checked_before_launch(L, name, template, rules):
    fn = getattr(L, name)
    for idx, boundary in rules.items():
        # every offset that leaves the boundary, at one byte and at half of it
        for off in sorted({1, boundary // 2}):
            if off == 0:
                continue
            args = []
            for k, a in enumerate(template):
                if isinstance(a, tuple):
                    addr = _base(a[1]) + (off if k == idx else 0)
                    args.append(ctypes.c_void_p(addr))
                else:
                    args.append(a)
            assert fn(*args) == EALIGN, (name, idx, off)


# The pointers each call needs (all but the optional status word and the
# stream), by argument index, for the same templates: on a non-empty shape a
# null in any of them is MXQ_ERR_INVALID_ARG before a launch.
_REQUIRED_POINTERS = {
    "mx_quantize": (0, 4, 5), "mx_dequantize": (0, 1, 4), "quantize_cache": (0, 1),
    "quantize_cache_packed": (0, 6, 7), "dequantize_cache_packed": (0, 1, 6),
    "mxfp4_grouped_mm": (0, 1, 2, 3, 9), "mxfp4_w4a4_grouped_mm": (0, 1, 2, 3, 4, 9),
    "nvfp4_w4a4_grouped_mm": (0, 1, 2, 3, 4, 5, 6, 11), "nvfp4_quantize": (0, 4, 5, 6, 7),
    "nvfp4_quantize_mse": (0, 4, 5, 6, 7), "nvfp4_quantize_noalloc": (0, 4, 5, 6),
    "nvfp4_dequantize": (0, 1, 2, 5), "mxq_debug_selftest": (0,),
}


@pytest.mark.parametrize("name,template,rules", _ALIGNED_POINTERS,
                         ids=["%s-%d" % (e[0], i) for i, e in enumerate(_ALIGNED_POINTERS)])
def test_every_required_pointer_is_checked_before_launch(L, name, template, rules):
    fn = getattr(L, name)
    for idx in _REQUIRED_POINTERS[name]:
        args = [ctypes.c_void_p(0 if k == idx else _base(a[1])) if isinstance(a, tuple) else a
                for k, a in enumerate(template)]
        assert fn(*args) == EARG, (name, idx)
