"""The C-ABI library on the CPU: it loads, exports every symbol include/attn_fwd.h
declares, and rejects bad arguments with the documented codes before any CUDA
call (no kernel runs here)."""
import ctypes
import os
import re

import pytest

import attention_forward_18_b200 as af

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_fwd.h")

# fake, never-dereferenced device addresses (16-byte aligned, far apart)
Q, K, V, O, L = 0x10000000, 0x20000000, 0x30000000, 0x40000000, 0x50000000


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(attn_\w+)\s*\(", text, re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(af.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(af.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_strerror():
    assert af.abi_version() == 1
    for code in range(0, -12, -1):
        msg = af.strerror(code)
        assert msg and msg != "unknown error code", code
    assert af.strerror(12345) == "unknown error code"


def call(q=Q, k=K, v=V, o=O, lse=L, B=1, H=2, Sq=128, Sk=128, D=64, causal=0,
         scale=0.125, dtype=af.ATTN_F16):
    return af.attn_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, causal, scale, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), af.ATTN_ERR_NULLPTR),
    (dict(k=None), af.ATTN_ERR_NULLPTR),
    (dict(v=None), af.ATTN_ERR_NULLPTR),
    (dict(o=None), af.ATTN_ERR_NULLPTR),
    (dict(dtype=2), af.ATTN_ERR_DTYPE),
    (dict(dtype=-1), af.ATTN_ERR_DTYPE),
    (dict(D=96), af.ATTN_ERR_HEADDIM),
    (dict(D=0), af.ATTN_ERR_HEADDIM),
    (dict(B=0), af.ATTN_ERR_SHAPE),
    (dict(H=-1), af.ATTN_ERR_SHAPE),
    (dict(Sq=0), af.ATTN_ERR_SHAPE),
    (dict(Sk=0), af.ATTN_ERR_SHAPE),
    (dict(Sq=(1 << 24) + 1), af.ATTN_ERR_SHAPE),
    (dict(B=1 << 13, H=1 << 12), af.ATTN_ERR_SHAPE),
    (dict(scale=float("nan")), af.ATTN_ERR_SCALE),
    (dict(scale=float("inf")), af.ATTN_ERR_SCALE),
    (dict(q=Q + 8), af.ATTN_ERR_ALIGN),
    (dict(o=O + 2), af.ATTN_ERR_ALIGN),
    (dict(lse=L + 2), af.ATTN_ERR_ALIGN),
    (dict(o=Q + 16), af.ATTN_ERR_ALIAS),
    (dict(o=V), af.ATTN_ERR_ALIAS),
    (dict(lse=K + 64), af.ATTN_ERR_ALIAS),
    (dict(lse=O + 1024), af.ATTN_ERR_ALIAS),
])
def test_argument_errors(kw, code):
    assert call(**kw) == code


def test_host_entry_checks_host_pointers():
    rc = af.attn_fwd_host(None, K, V, O, None, Q, K, V, O, L, 1, 1, 8, 8, 64, 0, 0.1,
                          af.ATTN_F16, None)
    assert rc == af.ATTN_ERR_NULLPTR


def test_status_rejects_null_out_pointer():
    assert af._lib.attn_fwd_status(None, None) == af.ATTN_ERR_NULLPTR


def test_valid_call_without_device_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    assert call() == af.ATTN_ERR_DEVICE


def test_binding_rejects_bad_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        af.attention(q, q, q)
    with pytest.raises(ValueError):
        af.attention(q[0], q[0], q[0])
