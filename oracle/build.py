"""Compile the scalar CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain gcc, no fast-math and no floating-point contraction, so every
operation in the oracle is the IEEE double operation written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mxq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
# The same source built with OpenMP: its row loops run on all host cores
# (the benchmark's all-core CPU baseline); the arithmetic is unchanged.
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")


def compile_to(src: str, out: str, openmp: bool = False) -> str:
    """Compile one oracle source file into a shared library at `out` (the
    flags of the oracle itself; the mutation tests build planted-mistake
    copies with it)."""
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra"] + (["-fopenmp"] if openmp else []) + \
          ["-o", tmp, src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False, openmp: bool = False) -> str:
    lib = LIB_OMP if openmp else LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    return compile_to(SRC, lib, openmp)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build(force="--force" in sys.argv, openmp=True))
