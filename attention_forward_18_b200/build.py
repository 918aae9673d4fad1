"""Build the CUDA library libattn_fwd.so in-tree with nvcc for sm_100a.

    python attention_forward_18_b200/build.py [--force] [--verbose-ptxas]

(run as a script: importing the package needs the library this builds)
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, f) for f in ("attn_fwd.cu", "row_softmax.cu", "gemm_bias_act.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("attn_fwd_kernel.cuh", "attn_fwd_wide_kernel.cuh", "attn_fwd_pair_kernel.cuh", "attn_merge.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", h) for h in ("attn_fwd.h", "row_softmax.h", "gemm_bias_act.h")]
LIB = os.path.join(HERE, "libattn_fwd.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
              "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O2", "-cudart", "static",
              "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def build(force=False, ptxas_verbose=False):
    """Compile when the library is missing or older than any source; returns its path."""
    stale = not os.path.exists(LIB) or any(
        os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if force or stale or ptxas_verbose:
        cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if ptxas_verbose else []),
               *SOURCES, "-o", LIB]
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv))
