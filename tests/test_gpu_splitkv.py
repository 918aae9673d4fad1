"""Split-KV pass (decode-shaped inputs) vs the fp64 oracle, element by element, through
the C ABI: partial results per KV range, merged by their log-sum-exp.  Same tolerances
as the whole pass (max |dO| <= 2e-2, max |dLSE| <= 1e-3)."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import O_TOL, compare
from workloads import make_qkv

pytestmark = pytest.mark.gpu


def run_split(q, k, v, causal, scale, n_splits=None, workspace=None, with_lse=True):
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_splitkv(dq, dk, dv, causal=causal, scale=scale, n_splits=n_splits,
                                  workspace=workspace, with_lse=with_lse)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    return (o.double().cpu().numpy(),
            lse.double().cpu().numpy() if lse is not None else None)


def check_split(B, H, Sq, Sk, D, dtype, causal, n_splits, seed, k_scale=1.0):
    scale = 1.0 / np.sqrt(D)
    q, k, v = make_qkv(B, H, Sq, Sk, D, dtype, seed, k_scale)
    o, lse = run_split(q, k, v, causal, scale, n_splits)
    o_ref, lse_ref = oracle.attn_ref(q.double().numpy(), k.double().numpy(),
                                     v.double().numpy(), causal, scale)
    return compare(o, lse, o_ref, lse_ref,
                   f"split B{B} H{H} Sq{Sq} Sk{Sk} D{D} {dtype} c{causal} n{n_splits}")


DECODE = [(1, 129), (1, 4096), (4, 1000), (16, 8191), (64, 2048), (128, 4097), (300, 3000)]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", DECODE)
def test_decode_shapes_default_splits(Sq, Sk, causal, dtype, D):
    check_split(2, 4, Sq, Sk, D, dtype, causal, None, seed=Sq * 13 + Sk)


@pytest.mark.parametrize("n_splits", [1, 2, 3, 7, 16, 32, 64, 1024])
def test_split_counts_including_empty_ranges(n_splits):
    """Sk = 1000 is 8 KV tiles: from 9 splits on, trailing ranges hold no tile and must
    contribute nothing."""
    check_split(1, 3, 16, 1000, 128, "bf16", False, n_splits, seed=n_splits)


@pytest.mark.parametrize("n_splits", [2, 5, 40])
def test_causal_ranges_a_row_cannot_see(n_splits):
    """Top-left mask with Sq < Sk: query i sees keys 0..i only, so every range past the
    query block is empty for all its rows (LSE_s = -inf) and the ranges in between are
    partly masked."""
    check_split(2, 2, 200, 6000, 64, "f16", True, n_splits, seed=40 + n_splits)


def test_long_context_decode():
    """One query per head against 32768 keys (256 KV tiles)."""
    check_split(1, 8, 1, 32768, 128, "bf16", False, None, seed=7, k_scale=3.0)


def test_single_split_is_the_whole_pass_bit_for_bit():
    """With one range the partial result is the whole-pass result and its merge weight
    is exactly 1, so O and LSE must equal attn_fwd's bit for bit."""
    q, k, v = make_qkv(2, 4, 300, 1500, 128, "bf16", 11)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    for causal in (False, True):
        o1, l1 = af.attention(dq, dk, dv, causal=causal)
        o2, l2 = af.attention_splitkv(dq, dk, dv, causal=causal, n_splits=1)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_workspace_garbage_and_reuse():
    """The workspace needs no initialisation: filled with NaN bytes first, then reused by
    a second call on other inputs; both results match the oracle and a repeat of the
    first call is bit-identical."""
    B, H, Sq, Sk, D = 1, 4, 64, 5000, 64
    n = 9
    nbytes = af.splitkv_workspace_bytes(B, H, Sq, D, n)
    ws = torch.full((nbytes + 4096,), 0xFF, dtype=torch.uint8, device="cuda")
    scale = 0.125
    qa, ka, va = make_qkv(B, H, Sq, Sk, D, "f16", 21)
    qb, kb, vb = make_qkv(B, H, Sq, Sk, D, "f16", 22)
    oa, la = run_split(qa, ka, va, True, scale, n, ws)
    ob, lb = run_split(qb, kb, vb, False, scale, n, ws)
    oa2, la2 = run_split(qa, ka, va, True, scale, n, ws)
    for (o, l, (q, k, v), c) in ((oa, la, (qa, ka, va), True), (ob, lb, (qb, kb, vb), False)):
        o_ref, l_ref = oracle.attn_ref(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy(), c, scale)
        compare(o, l, o_ref, l_ref, f"reuse causal={c}")
    assert np.array_equal(oa, oa2) and np.array_equal(la, la2)


def test_lse_pointer_may_be_null():
    q, k, v = make_qkv(1, 2, 8, 3000, 128, "bf16", 5)
    o, lse = run_split(q, k, v, False, 0.08, 4, with_lse=False)
    assert lse is None
    o_ref, _ = oracle.attn_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               False, 0.08)
    assert np.abs(o - o_ref).max() <= O_TOL


def test_workspace_too_small_is_rejected_on_device():
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 8, 3000, 128, "bf16", 5))
    need = af.splitkv_workspace_bytes(1, 2, 8, 128, 4)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    rc = af.attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None,
                             1, 2, 8, 3000, 128, 0, 0.1, af.ATTN_BF16, 4, ws.data_ptr(),
                             need - 1, None)
    assert rc == af.ATTN_ERR_WORKSPACE


@pytest.mark.parametrize("name", ["DEC1", "DEC2", "DEC3", "DEC4", "DEC5", "DEC6"])
def test_decode_workloads_in_bench_configuration(name):
    """The benchmark's decode workloads with the split count the benchmark uses (DEC5
    with grouped K/V heads through attn_fwd_ex): every row against the oracle (sampled
    rows for DEC3's 2048 rows x 64K keys)."""
    from workloads import DECODE_WORKLOADS, make_inputs, sample_rows
    w = DECODE_WORKLOADS[name]
    q, k, v = make_inputs(w)
    n = af.ex_default_splits(w.B, w.H, w.kv_heads, w.Sq, w.Sk, af.ATTN_MASK_NONE, w.D)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=af.ATTN_MASK_NONE, scale=w.scale, n_splits=n)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    o, lse = o.double().cpu().numpy(), lse.double().cpu().numpy()
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    if w.Sq <= 8:
        o_ref, lse_ref = oracle.attn_ref_ex(qd, kd, vd, oracle.NO_MASK, w.scale)
        compare(o, lse, o_ref, lse_ref, name)
    else:
        rows = sample_rows(w.B, w.H, w.Sq, 64, seed=w.seed)
        ro, rl = oracle.attn_ref_rows_ex(qd, kd, vd, rows, oracle.NO_MASK, w.scale)
        idx = tuple(np.array(rows).T)
        compare(o[idx], lse[idx], ro, rl, name)
