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
    for code in range(0, -13, -1):
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


W = 0x60000000  # fake 256-byte aligned workspace address


def split_call(n_splits=4, ws=W, ws_bytes=None, **kw):
    args = dict(q=Q, k=K, v=V, o=O, lse=L, B=1, H=2, Sq=64, Sk=4096, D=128, causal=0,
                scale=0.1, dtype=af.ATTN_BF16)
    args.update(kw)
    if ws_bytes is None:
        ws_bytes = af.splitkv_workspace_bytes(args["B"], args["H"], args["Sq"], args["D"],
                                              max(n_splits, 1))
    return af.attn_fwd_splitkv(args["q"], args["k"], args["v"], args["o"], args["lse"],
                               args["B"], args["H"], args["Sq"], args["Sk"], args["D"],
                               args["causal"], args["scale"], args["dtype"], n_splits, ws,
                               ws_bytes, None)


def test_splitkv_workspace_size_formula():
    # partial O (fp32, rounded up to 256 bytes) then partial LSE (fp32)
    B, H, Sq, D, S = 2, 3, 17, 64, 5
    o_part = -(-(S * B * H * Sq * D * 4) // 256) * 256
    assert af.splitkv_workspace_bytes(B, H, Sq, D, S) == o_part + S * B * H * Sq * 4
    assert af.splitkv_workspace_bytes(B, H, Sq, 96, S) == 0
    assert af.splitkv_workspace_bytes(B, H, Sq, D, 0) == 0
    assert af.splitkv_workspace_bytes(B, H, Sq, D, 1025) == 0


def test_splitkv_default_splits_in_range():
    # no device here: the library assumes 148 SMs
    s = af.splitkv_default_splits(1, 8, 16, 32768)
    assert 1 <= s <= 256
    assert af.splitkv_default_splits(1, 1, 1, 100) == 1      # a single KV tile
    assert af.splitkv_default_splits(0, 1, 1, 100) == 0
    # 16 heads x 1024 tiles: one round of 144 units of 114 tiles beats two rounds
    assert af.splitkv_default_splits(2, 8, 1, 131072) == 9
    # top-left causal with one query row: only key 0 is visible, nothing to split
    assert af.splitkv_default_splits(1, 8, 1, 131072, causal=True) == 1
    # many units already fill the SMs
    assert af.splitkv_default_splits(64, 32, 256, 256) == 1


@pytest.mark.parametrize("kw,code", [
    (dict(n_splits=0), af.ATTN_ERR_SHAPE),
    (dict(n_splits=1025), af.ATTN_ERR_SHAPE),
    (dict(ws=None), af.ATTN_ERR_NULLPTR),
    (dict(ws=W + 128), af.ATTN_ERR_ALIGN),
    (dict(ws_bytes=1024), af.ATTN_ERR_WORKSPACE),
    (dict(ws=Q + 4096), af.ATTN_ERR_ALIAS),
    (dict(ws=O - 256), af.ATTN_ERR_ALIAS),
    (dict(D=80), af.ATTN_ERR_HEADDIM),
])
def test_splitkv_argument_errors(kw, code):
    assert split_call(**kw) == code
