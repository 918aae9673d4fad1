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
    Hkv: int = 0        # K/V heads (grouped-query attention); 0 means H

    @property
    def kv_heads(self):
        return self.Hkv or self.H

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self):
        return TORCH_DTYPES[self.dtype]

    def flops(self, causal):
        return flops(self.B, self.H, self.Sq, self.Sk, self.D, causal)

    def io_bytes(self):
        if self.kv_heads != self.H:
            # Q read and O written per query head, K and V read per K/V head
            return (2 * self.B * self.D * (2 * self.H * self.Sq + 2 * self.kv_heads * self.Sk)
                    + 4 * self.B * self.H * self.Sq)
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
    "DEC5": Workload("DEC5", 8, 32, 1, 8192, 128, "bf16", (False,), 9, Hkv=8,
                     note="grouped heads: 32 query heads on 8 K/V heads, batch 8, 8K keys"),
    "DEC6": Workload("DEC6", 4, 16, 1, 16384, 256, "bf16", (False,), 32,
                     note="head dimension 256, batch of 4, one query row per head, 16K keys"),
}


# Wide head dimensions (the wide kernel: one 128-row query tile per CTA, 64-key KV
# tiles), non-causal and causal on the same tensors, same input recipe.
WIDE_WORKLOADS = {
    "WD192": Workload("WD192", 2, 16, 4096, 4096, 192, "bf16", (False, True), 30,
                      note="head dimension 192"),
    "WD256": Workload("WD256", 2, 16, 4096, 4096, 256, "bf16", (False, True), 31,
                      note="head dimension 256"),
}


# Chunked prefill with grouped K/V heads and the bottom-right causal mask: a chunk of
# 2048 new query rows attends to the 8192 keys of its context (the 6144 before it and
# itself, causally).
PREFILL_WORKLOADS = {
    "PRE1": Workload("PRE1", 1, 32, 2048, 8192, 128, "bf16", (True,), 10, Hkv=8,
                     note="chunked prefill: 2048 new rows, 8192-key context, 32 query "
                          "heads on 8 K/V heads, bottom-right causal"),
}


def visible_pairs(Sq, Sk, mask):
    """Number of (query, key) pairs a mask lets through per head: 0 none, 1 top-left
    causal (key j visible iff j <= i), 2 bottom-right (iff j <= i + Sk - Sq)."""
    if mask == 0:
        return Sq * Sk
    off = 0 if mask == 1 else Sk - Sq
    total = 0
    for i in range(Sq):
        total += max(0, min(Sk, i + off + 1))
    return total


@dataclass(frozen=True)
class RowWorkload:
    """A rows x n matrix for the standalone row softmax: i.i.d. N(0, 1) times `scale`
    (float32 from the seeded generator), rounded RN to `dtype`."""
    name: str
    rows: int
    n: int
    dtype: str          # "f16", "bf16" or "f32"
    seed: int
    scale: float = 1.0
    note: str = ""

    def io_bytes(self):
        """Algorithmic HBM bytes of one pass: x read once, y written once."""
        return 2 * self.rows * self.n * (4 if self.dtype == "f32" else 2)


# Row-softmax workloads (the pages give the step no sizes): attention-score rows,
# vocabulary-sized logits, and rows too long for one CTA's registers.
SOFTMAX_WORKLOADS = {
    "SMX1": RowWorkload("SMX1", 32768, 4096, "f16", 11, 4.0,
                        note="attention-score rows: 32768 rows of 4096, fp16"),
    "SMX2": RowWorkload("SMX2", 4096, 32000, "bf16", 12, 4.0,
                        note="vocabulary logits: 4096 rows of 32000, bf16"),
    "SMX3": RowWorkload("SMX3", 64, 1 << 20, "f32", 13, 8.0,
                        note="long rows: 64 rows of 2^20, fp32 (two-pass path)"),
}

TORCH_DTYPES_ALL = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def make_rows(rows, n, dtype, seed, scale=1.0):
    """Seeded rows x n matrix on the CPU in `dtype` ("f16", "bf16" or "f32")."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn((rows, n), generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(TORCH_DTYPES_ALL[dtype])



@dataclass(frozen=True)
class GemmWorkload:
    """C = act(A W^T + bias): A [M, K], W [N, K], bias [N], i.i.d. N(0, 1) float32 from
    the seeded generator in the order A, W, bias, A and W scaled by 1/sqrt(sqrt(K)) so
    the products stay O(1), rounded RN to `dtype`."""
    name: str
    M: int
    N: int
    K: int
    dtype: str          # "f16" or "bf16"
    act: int            # 0 none, 1 GELU, 2 ReLU
    seed: int
    note: str = ""

    def flops(self):
        return 2.0 * self.M * self.N * self.K


# GEMM workloads (the pages give the tutorial's GEMM no sizes): a square GEMM, an MLP
# up-projection of 4096 tokens, a short-K layer.
GEMM_WORKLOADS = {
    "GEMM1": GemmWorkload("GEMM1", 8192, 8192, 8192, "bf16", 1, 21,
                          note="square 8192^3, bias + GELU"),
    "GEMM2": GemmWorkload("GEMM2", 4096, 14336, 4096, "bf16", 1, 22,
                          note="MLP up-projection: 4096 tokens, 4096 -> 14336, bias + GELU"),
    "GEMM3": GemmWorkload("GEMM3", 8192, 8192, 1024, "f16", 2, 23,
                          note="short K: 8192 x 8192 x 1024, bias + ReLU, fp16"),
}


def make_gemm(M, N, K, dtype, seed):
    """Seeded A [M, K], W [N, K], bias [N] on the CPU in `dtype`."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    s = float(K) ** -0.25
    a = torch.randn((M, K), generator=g, dtype=torch.float32) * s
    w = torch.randn((N, K), generator=g, dtype=torch.float32) * s
    b = torch.randn((N,), generator=g, dtype=torch.float32)
    t = TORCH_DTYPES[dtype]
    return a.to(t), w.to(t), b.to(t)


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
    if w.kv_heads != w.H:
        # Q from the workload's seed, K and V (K/V heads only) from a second stream
        q, _, _ = make_qkv(w.B, w.H, w.Sq, 1, w.D, w.dtype, w.seed, w.k_scale)
        _, k, v = make_qkv(w.B, w.kv_heads, 1, w.Sk, w.D, w.dtype, w.seed + 100003, w.k_scale)
        return q, k, v
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
