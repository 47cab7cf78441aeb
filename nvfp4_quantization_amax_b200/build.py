"""Build libmxq.so (the C-ABI library of sm_100a kernels) in-tree.

    python -m nvfp4_quantization_amax_b200.build [--force] [--verbose] [--debug]

Every .cu under csrc/ is compiled for sm_100a only
(-gencode arch=compute_100a,code=sm_100a) with line info, without fast-math
(subnormals are kept: several results depend on them), and linked into
nvfp4_quantization_amax_b200/libmxq.so next to this file.  Object files go to
_build/ beside it.  nvcc cross-compiles, so no GPU is needed to build.

--debug builds the debug variant, libmxq_debug.so (objects in _build_debug/):
the same sources with MXQ_DEBUG_CHECKS, whose kernels test every indexed
access against its extent and record failures instead of touching memory.
"""
import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmxq.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libmxq_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  [os.path.join(INCLUDE, "mxq.h")])


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    flags = FLAGS + (["-DMXQ_DEBUG_CHECKS"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_dep = max(os.path.getmtime(p) for p in _deps())
    objs, jobs = [], []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        stale = (force or not os.path.exists(obj) or
                 os.path.getmtime(obj) < max(os.path.getmtime(src), newest_dep))
        if stale:
            jobs.append([NVCC] + ARCH + flags + (["-Xptxas", "-v"] if verbose else []) +
                        ["-c", src, "-o", obj])
    # translation units compile independently: one nvcc per source, in parallel
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        for f in [ex.submit(subprocess.check_call, cmd) for cmd in jobs]:
            f.result()
    if force or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib)
                                                for o in objs):
        tmp = lib + ".tmp%d" % os.getpid()
        subprocess.check_call([NVCC] + ARCH + ["-shared", "-o", tmp] + objs)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                debug="--debug" in sys.argv))
