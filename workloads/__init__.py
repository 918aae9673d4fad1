"""Seeded synthetic inputs for the attention forward pass.

This module is shared by the CUDA path's tests and benchmark and by the oracle's
tests.  It draws random numbers and holds the workload table; it contains none of
the attention arithmetic.

The tutorial pages measure on no dataset, so every workload is synthetic:
Q, K, V i.i.d. N(0, 1), drawn in float32 from a CPU ``torch.Generator`` seeded per
workload, in the fixed order q, k, v; a workload may scale K before rounding (the
"peaky" case multiplies K by 3 so the scores are N(0, 9)); the tensors are then
rounded to the workload's 16-bit type with round-to-nearest-even.  The oracle reads
those same rounded values upcast exactly to fp64.
"""
from dataclasses import dataclass
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    dtype: str          # "f16" or "bf16"
    causal: tuple       # the causal modes the workload runs (False, True or both)
    seed: int
    k_scale: float = 1.0
    note: str = ""

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self):
        return TORCH_DTYPES[self.dtype]

    def flops(self, causal):
        return flops(self.B, self.H, self.Sq, self.Sk, self.D, causal)

    def io_bytes(self):
        return io_bytes(self.B, self.H, self.Sq, self.Sk, self.D, 2)


TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}

# The five synthetic workloads (shapes, types, seeds and structure as stated for the
# benchmark of the fused forward pass).
WORKLOADS = {
    "C1": Workload("C1", 1, 2, 128, 128, 64, "f16", (False,), 0,
                   note="tiny non-causal case"),
    "C2": Workload("C2", 4, 16, 1024, 1024, 64, "f16", (False, True), 1,
                   note="non-causal and causal on the same tensors"),
    "C3": Workload("C3", 2, 32, 4096, 4096, 128, "bf16", (True,), 2,
                   note="causal"),
    "C4": Workload("C4", 8, 32, 2048, 2048, 128, "bf16", (False,), 3, k_scale=3.0,
                   note="non-causal, K scaled by 3 (peaky softmax)"),
    "C5": Workload("C5", 1, 16, 16384, 16384, 128, "bf16", (True,), 4,
                   note="long-context causal"),
}

# Decode-shaped workloads of the split-KV pass: few query rows per head against a long
# key sequence (the regime the pages' decode kernel serves), same input recipe.
DECODE_WORKLOADS = {
    "DEC1": Workload("DEC1", 1, 32, 1, 32768, 128, "bf16", (False,), 5,
                     note="one sequence, one query row per head, 32K keys"),
    "DEC2": Workload("DEC2", 8, 32, 1, 8192, 128, "bf16", (False,), 6,
                     note="batch of 8 sequences, one query row per head, 8K keys"),
    "DEC3": Workload("DEC3", 2, 16, 64, 65536, 128, "bf16", (False,), 7,
                     note="64 query rows per head (a block of drafted tokens), 64K keys"),
    "DEC4": Workload("DEC4", 16, 32, 1, 4096, 64, "f16", (False,), 8,
                     note="batch of 16, D=64, 4K keys"),
}


def flops(B, H, Sq, Sk, D, causal):
    """Counted FLOPs of one pass: 4*B*H*Sq*Sk*D (two GEMMs of 2 flops per
    multiply-add), halved for causal."""
    f = 4.0 * B * H * Sq * Sk * D
    return f / 2.0 if causal else f


def io_bytes(B, H, Sq, Sk, D, elem_bytes):
    """Algorithmic HBM bytes of one pass: Q, K, V read once, O written once (16-bit),
    plus the fp32 log-sum-exp."""
    return elem_bytes * B * H * D * (2 * Sq + 2 * Sk) + 4 * B * H * Sq


def make_qkv(B, H, Sq, Sk, D, dtype, seed, k_scale=1.0):
    """Seeded Q [B,H,Sq,D], K, V [B,H,Sk,D] on the CPU in the 16-bit `dtype`
    ("f16"/"bf16" or a torch dtype)."""
    if isinstance(dtype, str):
        dtype = TORCH_DTYPES[dtype]
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = torch.randn((B, H, Sq, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Sk, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Sk, D), generator=g, dtype=torch.float32)
    if k_scale != 1.0:
        k = k * k_scale
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_inputs(w: Workload):
    return make_qkv(w.B, w.H, w.Sq, w.Sk, w.D, w.dtype, w.seed, w.k_scale)


def sample_rows(B, H, Sq, n, seed, include_edges=True):
    """A seeded set of (b, h, i) query rows for spot checks: n random rows plus,
    when include_edges, the first and last row of the first and last head and the
    rows next to every 128-row tile boundary of one head."""
    g = torch.Generator(device="cpu").manual_seed(int(seed) + 7919)
    rows = []
    if include_edges:
        for (b, h) in {(0, 0), (B - 1, H - 1)}:
            rows += [(b, h, 0), (b, h, Sq - 1)]
        b, h = B // 2, H // 2
        for t in range(128, Sq, 128):
            rows += [(b, h, t - 1), (b, h, t)]
    if n > 0:
        bb = torch.randint(0, B, (n,), generator=g)
        hh = torch.randint(0, H, (n,), generator=g)
        ii = torch.randint(0, Sq, (n,), generator=g)
        rows += list(zip(bb.tolist(), hh.tolist(), ii.tolist()))
    seen, out = set(), []
    for r in rows:
        if r not in seen:
            seen.add(r)
            out.append(r)
    return out
