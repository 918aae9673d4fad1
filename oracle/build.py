"""Compile the fp64 CPU oracle (attn_ref.c) into oracle/liboracle_attn.so.

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

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def compile_oracle(src=SRC, out=LIB, extra=()):
    """Build `src` into the shared library `out`; returns `out`."""
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force=False):
    """Compile the oracle when the library is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_oracle()
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
