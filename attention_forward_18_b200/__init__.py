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

# Every symbol include/attn_fwd.h declares.
EXPORTS = ("attn_fwd", "attn_fwd_host", "attn_fwd_splitkv", "attn_fwd_splitkv_workspace_bytes",
           "attn_fwd_splitkv_default_splits", "attn_fwd_splitkv_noalloc", "attn_fwd_status",
           "attn_fwd_strerror", "attn_fwd_abi_version", "attn_fwd_debug")

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
_lib.attn_fwd_splitkv_default_splits.argtypes = [_i] * 5
_lib.attn_fwd_splitkv_default_splits.restype = _i
_lib.attn_fwd_splitkv_noalloc.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _vp]
_lib.attn_fwd_splitkv_noalloc.restype = _i
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


def splitkv_workspace_bytes(B, H, Sq, D, n_splits):
    return _lib.attn_fwd_splitkv_workspace_bytes(B, H, Sq, D, n_splits)


def splitkv_default_splits(B, H, Sq, Sk, causal=False):
    return _lib.attn_fwd_splitkv_default_splits(B, H, Sq, Sk, int(bool(causal)))


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


def _shape(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, S, D]")
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    if tuple(k.shape) != (B, H, Sk, D) or tuple(v.shape) != (B, H, Sk, D):
        raise ValueError("k and v must be [B, H, Sk, D] with q's B, H and D")
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
        n_splits = splitkv_default_splits(B, H, Sq, Sk, causal)
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
           "attention", "attention_splitkv", "attention_host", "splitkv_workspace_bytes",
           "splitkv_default_splits", "strerror", "abi_version", "AttnError", "ATTN_F16",
           "ATTN_BF16", "LIB_PATH", "EXPORTS"]
