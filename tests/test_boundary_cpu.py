"""The C-ABI library on the CPU: it loads, exports every symbol the headers in
include/ declare, and rejects bad arguments with the documented codes before any
CUDA call (no kernel runs here)."""
import ctypes
import glob
import os
import re

import pytest

import attention_forward_18_b200 as af

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))

# fake, never-dereferenced device addresses (16-byte aligned, far apart)
Q, K, V, O, L = 0x10000000, 0x20000000, 0x30000000, 0x40000000, 0x50000000


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, re.M))
    return sorted(names)


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(af.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(af.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_strerror():
    assert af.abi_version() == 2
    for code in range(0, -14, -1):
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
    (dict(D=72), af.ATTN_ERR_HEADDIM),
    (dict(D=0), af.ATTN_ERR_HEADDIM),
    (dict(D=160), af.ATTN_ERR_HEADDIM),
    (dict(D=224), af.ATTN_ERR_HEADDIM),
    (dict(D=320), af.ATTN_ERR_HEADDIM),
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
    assert af.splitkv_workspace_bytes(B, H, Sq, 72, S) == 0
    # head dimensions run zero-padded in the D = 128 kernel keep their own row size
    assert af.splitkv_workspace_bytes(B, H, Sq, 96, S) == (
        -(-(S * B * H * Sq * 96 * 4) // 256) * 256 + S * B * H * Sq * 4)
    # and so do the wide head dimensions
    for Dw in (192, 256):
        assert af.splitkv_workspace_bytes(B, H, Sq, Dw, S) == (
            -(-(S * B * H * Sq * Dw * 4) // 256) * 256 + S * B * H * Sq * 4)
    assert af.splitkv_workspace_bytes(B, H, Sq, 512, S) == 0
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


def test_default_splits_follow_the_kernel_geometry_of_D():
    # no device here: the library assumes 148 SMs.  4 single-row heads, 16384 keys: the
    # D = 128 kernel's 128 tiles of 128 keys fill 128 SMs best with 32 ranges; the wide
    # kernel's 256 tiles of 64 keys (D = 256 decode shapes) with 37 ranges of 7 tiles
    assert af.splitkv_default_splits(1, 4, 1, 16384, D=128) == 32
    assert af.splitkv_default_splits(1, 4, 1, 16384, D=256) == 37
    # 300 query rows at D = 256 run on CTA pairs (two SMs a unit): 4 units over 74 pairs
    # take 18 ranges, where 148 single-SM units would take 37
    assert af.splitkv_default_splits(1, 2, 300, 65536, D=128) == 37
    assert af.splitkv_default_splits(1, 2, 300, 65536, D=256) == 18
    # 64 single-row heads at D = 256: one round of 128 ranges of 128 tiles beats four
    # of 576 ranges of 29 (a 64-key range's fill is ~4 tiles)
    assert af.splitkv_default_splits(4, 16, 1, 16384, D=256) == 2
    assert af.ex_default_splits(1, 2, 2, 300, 65536, af.ATTN_MASK_NONE, D=192) == 18
    # head dimensions outside the library's set
    assert af.splitkv_default_splits(1, 4, 1, 16384, D=48) == 0
    assert af.ex_default_splits(1, 4, 4, 1, 16384, af.ATTN_MASK_NONE, D=512) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_splits=0), af.ATTN_ERR_SHAPE),
    (dict(n_splits=1025), af.ATTN_ERR_SHAPE),
    (dict(ws=None), af.ATTN_ERR_NULLPTR),
    (dict(ws=W + 128), af.ATTN_ERR_ALIGN),
    (dict(ws_bytes=1024), af.ATTN_ERR_WORKSPACE),
    (dict(ws=Q + 4096), af.ATTN_ERR_ALIAS),
    (dict(ws=O - 256), af.ATTN_ERR_ALIAS),
    (dict(D=144), af.ATTN_ERR_HEADDIM),
])
def test_splitkv_argument_errors(kw, code):
    assert split_call(**kw) == code


def ex_call(**kw):
    a = dict(q=Q, k=K, v=V, o=O, lse=L, B=2, H=8, H_kv=2, Sq=64, Sk=4096, D=128,
             mask=af.ATTN_MASK_NONE, scale=0.1, dtype=af.ATTN_BF16, n_splits=0, ws=None,
             ws_bytes=0)
    a.update(kw)
    return af.attn_fwd_ex(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["H_kv"],
                          a["Sq"], a["Sk"], a["D"], a["mask"], a["scale"], a["dtype"],
                          a["n_splits"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(mask=3), af.ATTN_ERR_MASK),
    (dict(mask=-1), af.ATTN_ERR_MASK),
    (dict(H_kv=3), af.ATTN_ERR_SHAPE),          # does not divide H
    (dict(H_kv=0), af.ATTN_ERR_SHAPE),
    (dict(H=64, H_kv=1, Sq=1 << 19), af.ATTN_ERR_SHAPE),   # 2^25 packed rows
    (dict(n_splits=-1), af.ATTN_ERR_SHAPE),
    (dict(n_splits=2), af.ATTN_ERR_NULLPTR),    # split pass without a workspace
    (dict(D=48), af.ATTN_ERR_HEADDIM),
    (dict(D=255), af.ATTN_ERR_HEADDIM),
    (dict(D=256, H=64, H_kv=1, Sq=1 << 19), af.ATTN_ERR_SHAPE),  # wide kernel, 2^25 rows
    (dict(o=K + 4096), af.ATTN_ERR_ALIAS),      # inside K (sized with H_kv heads)
])
def test_ex_argument_errors(kw, code):
    assert ex_call(**kw) == code


def test_ex_valid_arguments_reach_the_device_check():
    # no device here: valid arguments fail only at the device check
    assert ex_call() == af.ATTN_ERR_DEVICE
    assert ex_call(mask=af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT, H_kv=8) == af.ATTN_ERR_DEVICE


def test_ex_default_splits():
    assert af.ex_default_splits(2, 8, 8, 1, 131072) == af.splitkv_default_splits(2, 8, 1, 131072)
    # 4 query heads per K/V head are packed into one unit: fewer units, more splits
    assert af.ex_default_splits(1, 32, 8, 1, 32768) >= af.splitkv_default_splits(1, 32, 1, 32768)
    # bottom-right causal with one query row sees every key: split like non-causal
    assert (af.ex_default_splits(1, 8, 8, 1, 131072, af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT) ==
            af.ex_default_splits(1, 8, 8, 1, 131072, af.ATTN_MASK_NONE))
    assert af.ex_default_splits(1, 8, 3, 1, 100) == 0
    assert af.ex_default_splits(1, 8, 8, 1, 100, 5) == 0


@pytest.mark.parametrize("args,code", [
    ((Q, O, 4, 0, af.ATTN_F16), af.ATTN_ERR_SHAPE),
    ((Q, O, -1, 8, af.ATTN_F16), af.ATTN_ERR_SHAPE),
    ((Q, O, 4, (1 << 28) + 1, af.ATTN_F16), af.ATTN_ERR_SHAPE),
    ((Q, O, 4, 8, 3), af.ATTN_ERR_DTYPE),
    ((None, O, 4, 8, af.ATTN_F16), af.ATTN_ERR_NULLPTR),
    ((Q + 1, O, 4, 8, af.ATTN_F16), af.ATTN_ERR_ALIGN),
    ((Q, O + 2, 4, 8, af.SOFTMAX_F32), af.ATTN_ERR_ALIGN),
    ((Q, Q + 2, 4, 8, af.ATTN_F16), af.ATTN_ERR_ALIAS),     # partial overlap
    ((Q, O, 0, 8, af.ATTN_F16), af.ATTN_OK),                # no rows: nothing to do
    ((None, None, 0, 8, af.ATTN_F16), af.ATTN_OK),
    ((Q, Q, 4, 8, af.ATTN_F16), af.ATTN_ERR_DEVICE),        # in place is allowed
])
def test_row_softmax_argument_errors(args, code):
    x, y, rows, n, dt = args
    assert af.row_softmax_raw(x, y, rows, n, dt, None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(a=None), af.ATTN_ERR_NULLPTR),
    (dict(c=None), af.ATTN_ERR_NULLPTR),
    (dict(dtype=2), af.ATTN_ERR_DTYPE),
    (dict(act=3), af.ATTN_ERR_SHAPE),
    (dict(M=0), af.ATTN_ERR_SHAPE),
    (dict(N=12), af.ATTN_ERR_SHAPE),            # N not a multiple of 8
    (dict(K=100), af.ATTN_ERR_SHAPE),           # K not a multiple of 8
    (dict(a=Q + 8), af.ATTN_ERR_ALIGN),
    (dict(bias=V + 1), af.ATTN_ERR_ALIGN),
    (dict(c=Q + 64), af.ATTN_ERR_ALIAS),
    (dict(c=V - 16), af.ATTN_ERR_ALIAS),        # overlaps the bias
    (dict(), af.ATTN_ERR_DEVICE),               # valid: fails only at the device check
    (dict(bias=None), af.ATTN_ERR_DEVICE),
])
def test_gemm_argument_errors(kw, code):
    a = dict(a=Q, w=K, bias=V, c=O, M=300, N=512, K=1024, act=af.GEMM_ACT_GELU,
             dtype=af.ATTN_BF16)
    a.update(kw)
    assert af.gemm_bias_act_raw(a["a"], a["w"], a["bias"], a["c"], a["M"], a["N"], a["K"],
                                a["act"], a["dtype"], None) == code
