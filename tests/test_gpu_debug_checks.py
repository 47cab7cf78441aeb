"""The library's debug variant on the GPU.

libmxq_debug.so is the same sources built with MXQ_DEBUG_CHECKS: every kernel
tests the index of each global-memory access (and of the GEMMs' indexed
shared-memory stores) against the extent its launch was given, records a
failure (check id, index, extent) and skips the access, so nothing traps and
no out-of-range address is touched.  Here a child process loads it in place
of libmxq.so and runs the small parity cases of every entry point: results
must still equal the oracle's, and after every test no check may have
failed (tests/conftest.py).  A second child does the same for the
maximum-size cases.  A third runs the self-test, a checked store one element
past its declared extent, and reads the record back.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL_SHAPES = ["tests/test_gpu_parity.py", "tests/test_gpu_cache_packed.py",
                "tests/test_gpu_w4a4.py", "tests/test_gpu_nvfp4_mse.py",
                "tests/test_gpu_gemm_edges.py"]
NOT_SMALL = "not full_size and not eighteen and not full_expert and not timeout"


def debug_env():
    from nvfp4_quantization_amax_b200 import build

    env = dict(os.environ)
    env["MXQ_LIBRARY"] = build.build(debug=True)
    env["MXQ_EXPECT_CLEAN_CHECKS"] = "1"
    return env


def test_debug_variant_passes_the_small_parity_cases_without_a_failed_check():
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        "-k", NOT_SMALL] + SMALL_SHAPES,
                       cwd=ROOT, env=debug_env(), capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_debug_variant_at_the_largest_benchmark_size_without_a_failed_check():
    # the maximum-size cases (element indices past 2^31 in one call) with
    # every indexed access checked; both must run, not skip
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        "tests/test_gpu_max_size.py"],
                       cwd=ROOT, env=debug_env(), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert "2 passed" in r.stdout, r.stdout[-2000:]


SELFTEST = """
import torch
import nvfp4_quantization_amax_b200 as mxq
assert mxq.lib_path().endswith("libmxq_debug.so"), mxq.lib_path()
assert mxq.debug_checks() is None
w = torch.zeros(2, dtype=torch.int32, device="cuda")
mxq.debug_selftest(w)
torch.cuda.synchronize()
assert mxq.debug_checks() == (99, 1, 1)
assert mxq.debug_checks() is None  # reading clears the record
assert w.tolist() == [0, 0]        # the checked store was skipped
print("selftest ok")
"""


def test_debug_variant_records_a_failed_check():
    r = subprocess.run([sys.executable, "-c", SELFTEST], cwd=ROOT, env=debug_env(),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "selftest ok" in r.stdout, r.stdout + r.stderr
