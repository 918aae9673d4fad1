"""Compile the fp64 CPU oracles: attn_ref.c into oracle/liboracle_attn.so,
softmax_ref.c into oracle/liboracle_softmax.so and gemm_ref.c into
oracle/liboracle_gemm.so.

Test infrastructure only: the tests, the smoke check and the CPU-baseline leg of the
benchmark load the result; the product path never does.

Flags: -O2 with -ffp-contract=off and no fast-math, so each product and sum is one
IEEE fp64 rounding; OpenMP for the loops over heads / rows.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_ref.c")
LIB = os.path.join(HERE, "liboracle_attn.so")
SOFTMAX_SRC = os.path.join(HERE, "softmax_ref.c")
SOFTMAX_LIB = os.path.join(HERE, "liboracle_softmax.so")
GEMM_SRC = os.path.join(HERE, "gemm_ref.c")
GEMM_LIB = os.path.join(HERE, "liboracle_gemm.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def compile_oracle(src=SRC, out=LIB, extra=()):
    """Build `src` into the shared library `out`; returns `out`."""
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale(src, lib):
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


def build(force=False):
    """Compile the oracles when a library is missing or older than its source; returns
    the attention oracle's path."""
    if force or _stale(SRC, LIB):
        compile_oracle()
    if force or _stale(SOFTMAX_SRC, SOFTMAX_LIB):
        compile_oracle(SOFTMAX_SRC, SOFTMAX_LIB)
    if force or _stale(GEMM_SRC, GEMM_LIB):
        compile_oracle(GEMM_SRC, GEMM_LIB)
    return LIB


def build_softmax(force=False):
    build(force)
    return SOFTMAX_LIB


def build_gemm(force=False):
    build(force)
    return GEMM_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
