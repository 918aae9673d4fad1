"""Python binding of the B200 fused attention forward library (libattn_fwd.so).

Argument marshalling only: every step of the pass runs in the CUDA kernels behind
the C ABI declared in include/attn_fwd.h.  PyTorch supplies device memory and
streams.  There is no fallback: importing this package without the built library
raises ImportError, and every call on a machine without an sm_100 device returns
an error from the library (raised here as AttnError).

    import attention_forward_18_b200 as af
    o, lse = af.attention(q, k, v, causal=True)          # torch CUDA tensors [B,H,S,D]
    af.attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, Sq, Sk, D, causal, scale,
                af.ATTN_BF16, stream_ptr)                 # raw C-ABI call
"""
import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn_fwd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python attention_forward_18_b200/build.py` "
        "(there is no non-CUDA implementation)")

_lib = ctypes.CDLL(LIB_PATH)

ATTN_F16 = 0
ATTN_BF16 = 1
SOFTMAX_F32 = 2          # row_softmax only

GEMM_ACT_NONE = 0
GEMM_ACT_GELU = 1        # exact: 0.5 z (1 + erf(z / sqrt 2))
GEMM_ACT_RELU = 2

ATTN_OK = 0
ATTN_ERR_NULLPTR = -1
ATTN_ERR_ALIGN = -2
ATTN_ERR_SHAPE = -3
ATTN_ERR_HEADDIM = -4
ATTN_ERR_DTYPE = -5
ATTN_ERR_TENSORMAP = -6
ATTN_ERR_LAUNCH = -7
ATTN_ERR_TIMEOUT = -8
ATTN_ERR_SCALE = -9
ATTN_ERR_ALIAS = -10
ATTN_ERR_DEVICE = -11
ATTN_ERR_WORKSPACE = -12
ATTN_ERR_MASK = -13

ATTN_MASK_NONE = 0
ATTN_MASK_CAUSAL = 1                 # top-left: key j visible to query i iff j <= i
ATTN_MASK_CAUSAL_BOTTOM_RIGHT = 2    # iff j <= i + Sk - Sq

# Every symbol include/attn_fwd.h declares.
EXPORTS = ("attn_fwd", "attn_fwd_host", "attn_fwd_splitkv", "attn_fwd_splitkv_workspace_bytes",
           "attn_fwd_splitkv_default_splits", "attn_fwd_splitkv_noalloc", "attn_fwd_ex",
           "attn_fwd_ex_default_splits", "attn_fwd_status", "attn_fwd_strerror",
           "attn_fwd_abi_version", "attn_fwd_debug", "row_softmax", "gemm_bias_act",
           "gemm_bias_act_debug")

# Bytes of the library's own scratch behind attn_fwd_splitkv_noalloc.
SPLITKV_NOALLOC_SCRATCH_BYTES = 16 << 20

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_SIZES = [_i] * 6 + [_f, _i, _vp]   # B, H, Sq, Sk, D, causal, scale, dtype, stream

_lib.attn_fwd.argtypes = [_vp] * 5 + _SIZES
_lib.attn_fwd.restype = _i
_lib.attn_fwd_debug.argtypes = [_vp] * 5 + _SIZES + [ctypes.c_uint]
_lib.attn_fwd_debug.restype = _i
_lib.attn_fwd_host.argtypes = [_vp] * 10 + _SIZES
_lib.attn_fwd_host.restype = _i
_lib.attn_fwd_splitkv.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _vp, ctypes.c_size_t, _vp]
_lib.attn_fwd_splitkv.restype = _i
_lib.attn_fwd_splitkv_workspace_bytes.argtypes = [_i] * 5
_lib.attn_fwd_splitkv_workspace_bytes.restype = ctypes.c_size_t
_lib.attn_fwd_splitkv_default_splits.argtypes = [_i] * 6
_lib.attn_fwd_splitkv_default_splits.restype = _i
_lib.attn_fwd_splitkv_noalloc.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _vp]
_lib.attn_fwd_splitkv_noalloc.restype = _i
_lib.attn_fwd_ex.argtypes = [_vp] * 5 + [_i] * 7 + [_f, _i, _i, _vp, ctypes.c_size_t, _vp]
_lib.attn_fwd_ex.restype = _i
_lib.attn_fwd_ex_default_splits.argtypes = [_i] * 7
_lib.attn_fwd_ex_default_splits.restype = _i
_lib.gemm_bias_act.argtypes = [_vp] * 4 + [_i] * 5 + [_vp]
_lib.gemm_bias_act.restype = _i
_lib.gemm_bias_act_debug.argtypes = [_vp] * 4 + [_i] * 5 + [_vp, ctypes.c_uint]
_lib.gemm_bias_act_debug.restype = _i
_lib.row_softmax.argtypes = [_vp, _vp, ctypes.c_longlong, _i, _i, _vp]
_lib.row_softmax.restype = _i
_lib.attn_fwd_status.argtypes = [_vp, ctypes.POINTER(_i)]
_lib.attn_fwd_status.restype = _i
_lib.attn_fwd_strerror.argtypes = [_i]
_lib.attn_fwd_strerror.restype = ctypes.c_char_p
_lib.attn_fwd_abi_version.argtypes = []
_lib.attn_fwd_abi_version.restype = _i


class AttnError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


def strerror(code):
    return _lib.attn_fwd_strerror(int(code)).decode()


def abi_version():
    return _lib.attn_fwd_abi_version()


def _check(rc, where):
    if rc != ATTN_OK:
        raise AttnError(rc, where)
    return rc


# ------------------------------------------------------------------ raw C-ABI calls
def attn_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, causal, scale, dtype, stream):
    """The C call with integer pointers; returns its status code (no raise)."""
    return _lib.attn_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, int(causal), float(scale),
                         int(dtype), stream)


def attn_fwd_debug(q, k, v, o, lse, B, H, Sq, Sk, D, causal, scale, dtype, stream, flags):
    return _lib.attn_fwd_debug(q, k, v, o, lse, B, H, Sq, Sk, D, int(causal), float(scale),
                               int(dtype), stream, int(flags))


def attn_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev,
                  lse_dev, B, H, Sq, Sk, D, causal, scale, dtype, stream):
    return _lib.attn_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev,
                              o_dev, lse_dev, B, H, Sq, Sk, D, int(causal), float(scale),
                              int(dtype), stream)


def attn_fwd_splitkv(q, k, v, o, lse, B, H, Sq, Sk, D, causal, scale, dtype, n_splits,
                     workspace, workspace_bytes, stream):
    return _lib.attn_fwd_splitkv(q, k, v, o, lse, B, H, Sq, Sk, D, int(causal), float(scale),
                                 int(dtype), int(n_splits), workspace, int(workspace_bytes),
                                 stream)


def attn_fwd_splitkv_noalloc(q, k, v, o, lse, B, H, Sq, Sk, D, causal, scale, dtype, n_splits,
                             stream):
    """The split-KV pass into the library's own per-device scratch: no workspace
    argument, nothing allocated.  Returns the status code (no raise)."""
    return _lib.attn_fwd_splitkv_noalloc(q, k, v, o, lse, B, H, Sq, Sk, D, int(causal),
                                         float(scale), int(dtype), int(n_splits), stream)


def attn_fwd_ex(q, k, v, o, lse, B, H, H_kv, Sq, Sk, D, mask, scale, dtype, n_splits,
                workspace, workspace_bytes, stream):
    return _lib.attn_fwd_ex(q, k, v, o, lse, B, H, H_kv, Sq, Sk, D, int(mask), float(scale),
                            int(dtype), int(n_splits), workspace, int(workspace_bytes), stream)


def ex_default_splits(B, H, H_kv, Sq, Sk, mask=ATTN_MASK_NONE, D=128):
    return _lib.attn_fwd_ex_default_splits(B, H, H_kv, Sq, Sk, int(D), int(mask))


def splitkv_workspace_bytes(B, H, Sq, D, n_splits):
    return _lib.attn_fwd_splitkv_workspace_bytes(B, H, Sq, D, n_splits)


def splitkv_default_splits(B, H, Sq, Sk, causal=False, D=128):
    return _lib.attn_fwd_splitkv_default_splits(B, H, Sq, Sk, int(D), int(bool(causal)))


def attn_fwd_status(stream=None):
    """Synchronise `stream`, return and clear the device status word."""
    out = _i(0)
    _check(_lib.attn_fwd_status(_stream_ptr(stream), ctypes.byref(out)), "attn_fwd_status")
    return out.value


# ------------------------------------------------------------------ torch convenience
def _torch():
    import torch
    return torch


def _stream_ptr(stream):
    if stream is None:
        torch = _torch()
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float16:
        return ATTN_F16
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"q/k/v must be float16 or bfloat16, got {t.dtype}")


def _shape(q, k, v, grouped=False):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, S, D]")
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if not grouped and Hkv != H:
        raise ValueError("k and v must be [B, H, Sk, D] with q's B, H and D")
    if tuple(k.shape) != (B, Hkv, Sk, D) or tuple(v.shape) != (B, Hkv, Sk, D):
        raise ValueError("k and v must be [B, Hkv, Sk, D] with q's B and D")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    return B, H, Sq, Sk, D


def attention(q, k, v, causal=False, scale=None, out=None, lse=None, with_lse=True,
              stream=None):
    """O (and LSE) for CUDA tensors q [B,H,Sq,D], k, v [B,H,Sk,D] (fp16 or bf16).
    Outputs are allocated with torch unless given.  Returns (o, lse or None)."""
    torch = _torch()
    B, H, Sq, Sk, D = _shape(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    rc = _lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                       lse.data_ptr() if lse is not None else None, B, H, Sq, Sk, D,
                       int(bool(causal)), float(scale), _dtype_code(q), _stream_ptr(stream))
    _check(rc, "attn_fwd")
    return out, lse


def attention_splitkv(q, k, v, causal=False, scale=None, n_splits=None, out=None, lse=None,
                      with_lse=True, workspace=None, stream=None):
    """Split-KV pass (decode-shaped inputs): n_splits KV ranges per (query block, head)
    merged by their log-sum-exp.  The workspace is allocated with torch unless given.
    Returns (o, lse or None)."""
    torch = _torch()
    B, H, Sq, Sk, D = _shape(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if n_splits is None:
        n_splits = splitkv_default_splits(B, H, Sq, Sk, causal, D)
    nbytes = splitkv_workspace_bytes(B, H, Sq, D, n_splits)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    rc = _lib.attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr() if lse is not None else None, B, H, Sq, Sk, D,
                               int(bool(causal)), float(scale), _dtype_code(q), int(n_splits),
                               workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                               _stream_ptr(stream))
    _check(rc, "attn_fwd_splitkv")
    return out, lse


def attention_ex(q, k, v, mask=ATTN_MASK_NONE, scale=None, n_splits=0, out=None, lse=None,
                 with_lse=True, workspace=None, stream=None):
    """The general pass: k, v may have fewer heads than q (grouped-query attention:
    [B, Hkv, Sk, D], Hkv dividing H), `mask` is an ATTN_MASK_* value, `n_splits` 0 for
    the whole pass, None for the balanced split count, or a split count.  The split
    workspace is allocated with torch unless given.  Returns (o, lse or None)."""
    torch = _torch()
    B, H, Sq, Sk, D = _shape(q, k, v, grouped=True)
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if n_splits is None:
        n_splits = ex_default_splits(B, H, Hkv, Sq, Sk, mask, D)
    nbytes = splitkv_workspace_bytes(B, H, Sq, D, n_splits) if n_splits > 0 else 0
    if n_splits > 0 and workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    rc = _lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          lse.data_ptr() if lse is not None else None, B, H, Hkv, Sq, Sk, D,
                          int(mask), float(scale), _dtype_code(q), int(n_splits),
                          workspace.data_ptr() if workspace is not None else None,
                          workspace.numel() * workspace.element_size() if workspace is not None
                          else 0, _stream_ptr(stream))
    _check(rc, "attn_fwd_ex")
    return out, lse


def row_softmax_raw(x, y, rows, n, dtype, stream):
    """The C call row_softmax with integer pointers; returns its status code."""
    return _lib.row_softmax(x, y, int(rows), int(n), int(dtype), stream)


def row_softmax(x, out=None, stream=None):
    """Softmax along the last dimension of a contiguous CUDA tensor (fp16, bf16 or
    fp32).  `out` may be `x` (in place); allocated with torch unless given."""
    torch = _torch()
    codes = {torch.float16: ATTN_F16, torch.bfloat16: ATTN_BF16, torch.float32: SOFTMAX_F32}
    if x.dtype not in codes:
        raise TypeError(f"x must be float16, bfloat16 or float32, got {x.dtype}")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if out is None:
        out = torch.empty_like(x)
    n = x.shape[-1] if x.dim() else 1
    rows = x.numel() // n if n else 0
    _check(_lib.row_softmax(x.data_ptr(), out.data_ptr(), rows, n, codes[x.dtype],
                            _stream_ptr(stream)), "row_softmax")
    return out


def gemm_bias_act_raw(a, w, bias, c, M, N, K, act, dtype, stream, flags=0):
    """The C call gemm_bias_act (gemm_bias_act_debug when flags) with integer
    pointers; returns its status code."""
    if flags:
        return _lib.gemm_bias_act_debug(a, w, bias, c, M, N, K, int(act), int(dtype), stream,
                                        int(flags))
    return _lib.gemm_bias_act(a, w, bias, c, M, N, K, int(act), int(dtype), stream)


def gemm_bias_act(a, w, bias=None, act=GEMM_ACT_NONE, out=None, stream=None):
    """C = act(a @ w.T + bias) for CUDA tensors a [M, K], w [N, K], bias [N] or None
    (one 16-bit dtype); N and K multiples of 8.  Returns C [M, N]."""
    torch = _torch()
    if a.dim() != 2 or w.dim() != 2 or a.shape[1] != w.shape[1]:
        raise ValueError("a must be [M, K] and w [N, K]")
    M, K = a.shape
    N = w.shape[0]
    if bias is not None and (bias.shape != (N,) or bias.dtype != a.dtype):
        raise ValueError("bias must be [N] of a's dtype")
    if w.dtype != a.dtype:
        raise TypeError("a and w must share one dtype")
    for t in (a, w) + ((bias,) if bias is not None else ()):
        if not t.is_contiguous():
            raise ValueError("a, w, bias must be contiguous")
    if out is None:
        out = torch.empty((M, N), dtype=a.dtype, device=a.device)
    _check(_lib.gemm_bias_act(a.data_ptr(), w.data_ptr(),
                              bias.data_ptr() if bias is not None else None, out.data_ptr(),
                              M, N, K, int(act), _dtype_code(a), _stream_ptr(stream)),
           "gemm_bias_act")
    return out


def attention_host(q, k, v, staging, causal=False, scale=None, out=None, lse=None,
                   stream=None):
    """The pass from (pinned) host tensors through attn_fwd_host.  `staging` is a tuple
    (q_dev, k_dev, v_dev, o_dev, lse_dev) of device tensors of the matching shapes.
    The copies and the kernel are queued on `stream`; synchronise before reading."""
    torch = _torch()
    B, H, Sq, Sk, D = _shape(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q, pin_memory=True)
    qd, kd, vd, od, ld = staging
    rc = _lib.attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr() if lse is not None else None,
                            qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                            ld.data_ptr() if ld is not None else None, B, H, Sq, Sk, D,
                            int(bool(causal)), float(scale), _dtype_code(q),
                            _stream_ptr(stream))
    _check(rc, "attn_fwd_host")
    return out, lse


__all__ = ["attn_fwd", "attn_fwd_host", "attn_fwd_splitkv", "attn_fwd_splitkv_noalloc",
           "attn_fwd_status", "attn_fwd_debug", "SPLITKV_NOALLOC_SCRATCH_BYTES",
           "attention", "attention_splitkv", "attention_ex", "attention_host", "attn_fwd_ex",
           "ex_default_splits", "ATTN_MASK_NONE", "ATTN_MASK_CAUSAL",
           "ATTN_MASK_CAUSAL_BOTTOM_RIGHT", "splitkv_workspace_bytes",
           "splitkv_default_splits", "strerror", "abi_version", "AttnError", "ATTN_F16",
           "ATTN_BF16", "SOFTMAX_F32", "row_softmax", "row_softmax_raw", "gemm_bias_act",
           "gemm_bias_act_raw", "GEMM_ACT_NONE", "GEMM_ACT_GELU", "GEMM_ACT_RELU", "LIB_PATH",
           "EXPORTS"]
