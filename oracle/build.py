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


def compile_to(src: str, out: str) -> str:
    """Compile one oracle source file into a shared library at `out` (the
    flags of the oracle itself; the mutation tests build planted-mistake
    copies with it)."""
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
