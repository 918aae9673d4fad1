"""fp64 CPU oracle for the fused attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or calls it, and shares no code with it.

The arithmetic lives in ``attn_ref.c`` (plain C, fp64, libm ``exp``/``log``, no
fast-math); this module only marshals numpy arrays through ctypes.  It follows the
softmax-attention definition that the TileLang tutorial's FlashAttention section
validates against (pro.edgex.exchange summary, FlashAttention paragraph; datastack.it,
"Cosa copre il tutorial": causal and non-causal):

    O = softmax(scale * Q K^T  [+ causal mask]) V
    LSE_i = ln sum_j exp(scale * q_i . k_j)     (over the unmasked j)

The causal mask is top-left aligned (key j visible to query i iff j <= i) unless
``mask=CAUSAL_BOTTOM_RIGHT`` (j <= i + Sk - Sq; a row that sees no key gets O = 0,
LSE = -inf).  K and V may have fewer heads than Q (``Hkv`` divides ``H``; query head
h reads K/V head h // (H // Hkv)).  Both are the library's options beyond the pages.

Pins (see tests/test_oracle_pins.py): closed forms (Sk = 1, Q = 0, constant V,
causal row 0, one-hot attention), invariants (row sums, permutation and shift
invariance), hand-derived tiny cases, and PyTorch's float64 math SDPA on the CPU.
"""
import ctypes
import os

import numpy as np

from . import build as _build

NO_MASK = 0
CAUSAL_TOP_LEFT = 1
CAUSAL_BOTTOM_RIGHT = 2

ORACLE_OK = 0
ORACLE_ERR_ARGS = 1
ORACLE_ERR_NOMEM = 2
ORACLE_ERR_ROWSUM = 3

_LIB = None


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.c_long
    lib.attn_ref_f64.argtypes = [dp, dp, dp, dp, dp, dp, lp, lp, lp, lp, lp,
                                 ctypes.c_int, ctypes.c_double]
    lib.attn_ref_f64.restype = ctypes.c_int
    lib.attn_ref_rows_f64.argtypes = [dp, dp, dp, ctypes.POINTER(ctypes.c_int64), lp,
                                      dp, dp, lp, lp, lp, lp, lp, ctypes.c_int,
                                      ctypes.c_double]
    lib.attn_ref_rows_f64.restype = ctypes.c_int
    lib.attn_ref_ex_f64.argtypes = [dp, dp, dp, dp, dp, dp, lp, lp, lp, lp, lp, lp,
                                    ctypes.c_int, ctypes.c_double]
    lib.attn_ref_ex_f64.restype = ctypes.c_int
    lib.attn_ref_rows_ex_f64.argtypes = [dp, dp, dp, ctypes.POINTER(ctypes.c_int64), lp,
                                         dp, dp, lp, lp, lp, lp, lp, lp, ctypes.c_int,
                                         ctypes.c_double]
    lib.attn_ref_rows_ex_f64.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def load(path=None):
    """Load (building first if needed) the oracle library, or the one at `path`."""
    global _LIB
    if path is not None:
        return _bind(path)
    if _LIB is None:
        _LIB = _bind(_build.build())
    return _LIB


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads(lib=None):
    return (lib or load()).oracle_num_threads()


def attn_ref(q, k, v, causal, scale, return_probs=False, lib=None):
    """Whole problem.  q: [B,H,Sq,D], k, v: [B,H,Sk,D] (any real dtype, upcast
    exactly to fp64).  Returns (O [B,H,Sq,D], LSE [B,H,Sq]) in fp64, plus the
    probability matrices [B,H,Sq,Sk] when return_probs."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    if k.shape != (B, H, Sk, D) or v.shape != (B, H, Sk, D):
        raise ValueError("k and v must be [B,H,Sk,D] with q's B, H, D")
    o = np.empty((B, H, Sq, D), dtype=np.float64)
    lse = np.empty((B, H, Sq), dtype=np.float64)
    p = np.empty((B, H, Sq, Sk), dtype=np.float64) if return_probs else None
    rc = lib.attn_ref_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                          _ptr(p) if p is not None else None,
                          B, H, Sq, Sk, D, int(bool(causal)), float(scale))
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle attn_ref_f64 failed with code {rc}")
    return (o, lse, p) if return_probs else (o, lse)


def attn_ref_rows(q, k, v, rows, causal, scale, lib=None):
    """Selected query rows only.  rows: int array [n, 3] of (b, h, i).
    Returns (O [n, D], LSE [n]) in fp64."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.attn_ref_rows_f64(_ptr(q), _ptr(k), _ptr(v),
                               rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
                               _ptr(o), _ptr(lse), B, H, Sq, Sk, D,
                               int(bool(causal)), float(scale))
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle attn_ref_rows_f64 failed with code {rc}")
    return o, lse


def _mask_code(causal, mask):
    if mask is not None:
        if mask not in (NO_MASK, CAUSAL_TOP_LEFT, CAUSAL_BOTTOM_RIGHT):
            raise ValueError(f"unknown mask {mask}")
        return int(mask)
    return CAUSAL_TOP_LEFT if causal else NO_MASK


def attn_ref_ex(q, k, v, mask=None, scale=1.0, causal=False, return_probs=False, lib=None):
    """Whole problem with the extended options: k, v [B,Hkv,Sk,D] with Hkv dividing
    q's H; `mask` one of NO_MASK, CAUSAL_TOP_LEFT, CAUSAL_BOTTOM_RIGHT (or None: taken
    from `causal`).  Returns (O, LSE[, P]) in fp64 like attn_ref."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Sk, D) or v.shape != (B, Hkv, Sk, D):
        raise ValueError("k and v must be [B,Hkv,Sk,D] with q's B and D")
    o = np.empty((B, H, Sq, D), dtype=np.float64)
    lse = np.empty((B, H, Sq), dtype=np.float64)
    p = np.empty((B, H, Sq, Sk), dtype=np.float64) if return_probs else None
    rc = lib.attn_ref_ex_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(p) if p is not None else None,
                             B, H, Hkv, Sq, Sk, D, _mask_code(causal, mask), float(scale))
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle attn_ref_ex_f64 failed with code {rc}")
    return (o, lse, p) if return_probs else (o, lse)


def attn_ref_rows_ex(q, k, v, rows, mask=None, scale=1.0, causal=False, lib=None):
    """Selected rows with the extended options (see attn_ref_ex)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.attn_ref_rows_ex_f64(_ptr(q), _ptr(k), _ptr(v),
                                  rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
                                  _ptr(o), _ptr(lse), B, H, Hkv, Sq, Sk, D,
                                  _mask_code(causal, mask), float(scale))
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle attn_ref_rows_ex_f64 failed with code {rc}")
    return o, lse


# ------------------------------------------------------------------ row softmax
_SOFTMAX_LIB = None


def load_softmax(path=None):
    """Load (building first if needed) the row-softmax oracle, or the one at `path`."""
    global _SOFTMAX_LIB
    if path is None and _SOFTMAX_LIB is not None:
        return _SOFTMAX_LIB
    lib = ctypes.CDLL(path or _build.build_softmax())
    dp = ctypes.POINTER(ctypes.c_double)
    lib.softmax_ref_f64.argtypes = [dp, dp, ctypes.c_long, ctypes.c_long]
    lib.softmax_ref_f64.restype = ctypes.c_int
    lib.softmax_ref_num_threads.argtypes = []
    lib.softmax_ref_num_threads.restype = ctypes.c_int
    if path is None:
        _SOFTMAX_LIB = lib
    return lib


def softmax_ref(x, lib=None):
    """Row-wise softmax over the last axis of `x` (any real dtype, upcast exactly to
    fp64): y = exp(x - max) / sum exp(x - max).  Returns fp64 of x's shape.  Follows
    the fused-softmax paragraph of the pro.edgex.exchange summary of the tutorial."""
    lib = lib or load_softmax()
    x = _f64(x)
    n = x.shape[-1] if x.ndim else 1
    rows = x.size // n if n else 0
    y = np.empty_like(x)
    rc = lib.softmax_ref_f64(_ptr(x), _ptr(y), rows, n)
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle softmax_ref_f64 failed with code {rc}")
    return y


# ------------------------------------------------------------------ GEMM + bias + act
ACT_NONE = 0
ACT_GELU = 1
ACT_RELU = 2
_GEMM_LIB = None


def load_gemm(path=None):
    """Load (building first if needed) the GEMM oracle, or the one at `path`."""
    global _GEMM_LIB
    if path is None and _GEMM_LIB is not None:
        return _GEMM_LIB
    lib = ctypes.CDLL(path or _build.build_gemm())
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.c_long
    lib.gemm_bias_act_ref_f64.argtypes = [dp, dp, dp, dp, lp, lp, lp, ctypes.c_int]
    lib.gemm_bias_act_ref_f64.restype = ctypes.c_int
    lib.gemm_ref_num_threads.argtypes = []
    lib.gemm_ref_num_threads.restype = ctypes.c_int
    if path is None:
        _GEMM_LIB = lib
    return lib


def gemm_bias_act_ref(a, w, bias=None, act=ACT_NONE, lib=None):
    """C = act(A W^T + bias) in fp64: a [M,K], w [N,K], bias [N] or None (any real
    dtype, upcast exactly).  act: ACT_NONE, ACT_GELU (exact, erf form) or ACT_RELU.
    Follows the GEMM-with-epilogue step of the tutorial (pro.edgex.exchange summary:
    bias + GELU; comrad404.com summary: ReLU or bias)."""
    lib = lib or load_gemm()
    a, w = _f64(a), _f64(w)
    M, K = a.shape
    N = w.shape[0]
    if w.shape != (N, K):
        raise ValueError("w must be [N, K] with a's K")
    b = _f64(bias) if bias is not None else None
    if b is not None and b.shape != (N,):
        raise ValueError("bias must be [N]")
    c = np.empty((M, N), dtype=np.float64)
    rc = lib.gemm_bias_act_ref_f64(_ptr(a), _ptr(w), _ptr(b) if b is not None else None,
                                   _ptr(c), M, N, K, int(act))
    if rc != ORACLE_OK:
        raise RuntimeError(f"oracle gemm_bias_act_ref_f64 failed with code {rc}")
    return c


__all__ = ["gemm_bias_act_ref", "load_gemm", "ACT_NONE", "ACT_GELU", "ACT_RELU",
           "softmax_ref", "load_softmax", "attn_ref", "attn_ref_rows", "attn_ref_ex", "attn_ref_rows_ex", "load",
           "num_threads", "NO_MASK", "CAUSAL_TOP_LEFT", "CAUSAL_BOTTOM_RIGHT"]
