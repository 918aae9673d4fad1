"""attn_fwd_ex vs the fp64 oracle, element by element, through the C ABI: grouped K/V
heads (query head h reads K/V head h // (H / Hkv)), the bottom-right causal mask
(rows that see no key: O = 0, LSE = -inf), each with the whole pass and the split pass.
Tolerances as everywhere: max |dO| <= 2e-2, max |dLSE| <= 1e-3."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import LSE_TOL, O_TOL
from workloads import make_qkv

pytestmark = pytest.mark.gpu

MASKS = {"none": af.ATTN_MASK_NONE, "topleft": af.ATTN_MASK_CAUSAL,
         "bottomright": af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT}


def make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed):
    """Seeded inputs with Hkv K/V heads (the shared generator, K/V drawn per K/V head)."""
    q, _, _ = make_qkv(B, H, Sq, 1, D, dtype, seed)
    _, k, v = make_qkv(B, Hkv, 1, Sk, D, dtype, seed + 100003)
    return q, k, v


def compare_ex(o, lse, o_ref, lse_ref, what):
    assert np.isfinite(o).all(), what
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: empty rows differ"
    assert (o[empty] == 0).all(), f"{what}: O of an empty row is not 0"
    do = np.abs(o - o_ref).max()
    dl = np.abs(lse[~empty] - lse_ref[~empty]).max() if (~empty).any() else 0.0
    assert do <= O_TOL and dl <= LSE_TOL, f"{what}: max dO {do:.3e} max dLSE {dl:.3e}"


def check(B, H, Hkv, Sq, Sk, D, dtype, mask, n_splits, seed):
    q, k, v = make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed)
    scale = 1.0 / np.sqrt(D)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=MASKS[mask], scale=scale, n_splits=n_splits)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), MASKS[mask], scale)
    compare_ex(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
               f"B{B} H{H}/{Hkv} Sq{Sq} Sk{Sk} D{D} {dtype} {mask} n{n_splits}")


BR_SHAPES = [(1, 1), (1, 777), (64, 1000), (200, 6000), (300, 300), (129, 257),
             (400, 150), (1000, 129), (300, 1)]


@pytest.mark.parametrize("D,dtype", [(64, "f16"), (128, "bf16")])
@pytest.mark.parametrize("n_splits", [0, None])
@pytest.mark.parametrize("Sq,Sk", BR_SHAPES)
def test_bottom_right_mask(Sq, Sk, n_splits, D, dtype):
    """Sq < Sk (decode-like: the last query sees all keys), Sq = Sk (equal to top-left),
    Sq > Sk (the first Sq - Sk rows see nothing), whole pass and balanced splits."""
    check(2, 3, 3, Sq, Sk, D, dtype, "bottomright", n_splits, seed=Sq * 3 + Sk)


GQA = [(8, 1), (8, 2), (8, 4), (6, 3), (32, 8)]


@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
@pytest.mark.parametrize("H,Hkv", GQA)
@pytest.mark.parametrize("Sq,Sk", [(1, 3000), (5, 700), (100, 1000), (300, 300)])
def test_grouped_heads_whole(Sq, Sk, H, Hkv, mask):
    """Packed query tiles span head boundaries (e.g. Sq = 100: a 128-row tile holds
    one head's 100 rows and 28 of the next), so causal masks are per position."""
    check(2, H, Hkv, Sq, Sk, 128, "bf16", mask, 0, seed=H * 100 + Hkv * 10 + Sq)


@pytest.mark.parametrize("mask", ["none", "bottomright"])
@pytest.mark.parametrize("H,Hkv", GQA)
@pytest.mark.parametrize("n_splits", [None, 3, 17])
def test_grouped_heads_split(n_splits, H, Hkv, mask):
    """Decode with grouped heads: one query row per head, 8K keys, split KV."""
    check(2, H, Hkv, 1, 8192, 64, "f16", mask, n_splits, seed=H + Hkv + (n_splits or 0))


def test_plain_entry_points_equal_the_general_one():
    """attn_fwd / attn_fwd_splitkv are attn_fwd_ex with H_kv = H and the top-left mask,
    bit for bit."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 300, 1100, 128, "bf16", 9))
    for causal in (False, True):
        mask = af.ATTN_MASK_CAUSAL if causal else af.ATTN_MASK_NONE
        o1, l1 = af.attention(q, k, v, causal=causal)
        o2, l2 = af.attention_ex(q, k, v, mask=mask)
        o3, l3 = af.attention_splitkv(q, k, v, causal=causal, n_splits=4)
        o4, l4 = af.attention_ex(q, k, v, mask=mask, n_splits=4)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        assert torch.equal(o3, o4) and torch.equal(l3, l4)


def test_grouped_heads_equal_repeated_heads():
    """GQA with K/V repeated per query head (plain multi-head) gives the same result:
    the head mapping is the only difference."""
    B, H, Hkv, Sq, Sk, D = 2, 8, 2, 77, 900, 64
    q, k, v = (t.cuda() for t in make_gqa(B, H, Hkv, Sq, Sk, D, "f16", 13))
    ke, ve = (t.repeat_interleave(H // Hkv, dim=1).contiguous() for t in (k, v))
    for mask in MASKS.values():
        o1, l1 = af.attention_ex(q, k, v, mask=mask)
        o2, l2 = af.attention_ex(q, ke, ve, mask=mask)
        torch.cuda.synchronize()
        assert (o1.float() - o2.float()).abs().max().item() <= O_TOL
        assert (l1 - l2).abs().max().item() <= LSE_TOL


def test_prefill_workload_in_bench_configuration():
    """The benchmark's chunked-prefill workload (grouped heads, bottom-right causal) at
    full size: sampled rows against the oracle."""
    from workloads import PREFILL_WORKLOADS, make_inputs, sample_rows
    w = PREFILL_WORKLOADS["PRE1"]
    q, k, v = make_inputs(w)
    o, lse = af.attention_ex(q.cuda(), k.cuda(), v.cuda(), mask=af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT,
                             scale=w.scale)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    rows = sample_rows(w.B, w.H, w.Sq, 48, seed=w.seed)
    ro, rl = oracle.attn_ref_rows_ex(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                     rows, oracle.CAUSAL_BOTTOM_RIGHT, w.scale)
    idx = tuple(np.array(rows).T)
    compare_ex(o.double().cpu().numpy()[idx], lse.double().cpu().numpy()[idx], ro, rl, "PRE1")


@pytest.mark.parametrize("scale", [-0.2, 0.0])
@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
@pytest.mark.parametrize("n_splits", [0, 3])
def test_negative_and_zero_scale_on_every_path(n_splits, mask, scale):
    """The negative-scale and zero-scale handling on the split, grouped-head, general
    causal and decode instantiations (a decode shape: 4 packed rows per K/V head) and on
    a longer prefill shape."""
    for (Sq, Sk) in ((1, 2000), (300, 700)):
        q, k, v = make_gqa(2, 8, 2, Sq, Sk, 64, "f16", seed=Sq + Sk)
        dq, dk, dv = (t.cuda() for t in (q, k, v))
        o, lse = af.attention_ex(dq, dk, dv, mask=MASKS[mask], scale=scale, n_splits=n_splits)
        torch.cuda.synchronize()
        assert af.attn_fwd_status() == 0
        o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), MASKS[mask], scale)
        compare_ex(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                   f"scale {scale} mask {mask} splits {n_splits} Sq {Sq}")


@pytest.mark.parametrize("D", [80, 96, 112])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("case", ["whole_nc", "whole_causal", "split_decode", "gqa_br",
                                  "ragged"])
def test_padded_head_dims(case, dtype, D):
    """Head dimensions 80, 96 and 112 run in the D = 128 kernel with the missing
    columns read as zeros; every path against the oracle."""
    if case == "whole_nc":
        check(2, 3, 3, 300, 500, D, dtype, "none", 0, seed=D)
    elif case == "whole_causal":
        check(2, 3, 3, 500, 500, D, dtype, "topleft", 0, seed=D + 1)
    elif case == "split_decode":
        check(2, 4, 4, 1, 5000, D, dtype, "none", None, seed=D + 2)
    elif case == "gqa_br":
        check(1, 8, 2, 40, 3000, D, dtype, "bottomright", 5, seed=D + 3)
    else:
        check(1, 2, 2, 129, 257, D, dtype, "none", 0, seed=D + 4)
