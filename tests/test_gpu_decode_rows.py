"""Decode shapes of at most a few packed query rows per K/V head (the kernel's decode
form: every row in one query tile, both softmax warpgroups on alternate KV tiles, their
two partial results merged in the epilogue) vs the fp64 oracle, element by element,
through the C ABI.  Every mask, grouped heads, the whole pass and split passes (empty
ranges included), key counts that end inside and on the edge of a tile, every head
dimension of the D <= 128 kernel, negative, zero and large scales, running maxima that
rise tile after tile.  Tolerances as everywhere: max |dO| <= 2e-2, max |dLSE| <= 1e-3."""
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


def make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed, k_scale=1.0):
    q, _, _ = make_qkv(B, H, Sq, 1, D, dtype, seed)
    _, k, v = make_qkv(B, Hkv, 1, Sk, D, dtype, seed + 7919, k_scale)
    return q, k, v


def check(B, H, Hkv, Sq, Sk, D, dtype, mask, n_splits, seed, scale=None, k_scale=1.0):
    q, k, v = make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed, k_scale)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=MASKS[mask], scale=scale, n_splits=n_splits)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    o, lse = o.double().cpu().numpy(), lse.double().cpu().numpy()
    o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), MASKS[mask], scale)
    what = f"B{B} H{H}/{Hkv} Sq{Sq} Sk{Sk} D{D} {dtype} {mask} n{n_splits} scale {scale}"
    assert np.isfinite(o).all(), what
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: empty rows differ"
    assert (o[empty] == 0).all(), f"{what}: O of an empty row is not 0"
    do = float(np.abs(o - o_ref).max())
    dl = float(np.abs(lse[~empty] - lse_ref[~empty]).max()) if (~empty).any() else 0.0
    assert do <= O_TOL and dl <= LSE_TOL, f"{what}: max dO {do:.3e} max dLSE {dl:.3e}"
    return do, dl


# (H, Hkv, Sq): packed rows g * Sq from 1 to 10
ROWS = [(4, 4, 1), (4, 4, 2), (3, 3, 5), (2, 2, 8), (8, 4, 1), (8, 2, 1), (16, 2, 1),
        (4, 2, 3), (8, 2, 2), (6, 2, 3), (4, 2, 5)]


@pytest.mark.parametrize("mask", ["none", "bottomright", "topleft"])
@pytest.mark.parametrize("n_splits", [0, None, 3])
@pytest.mark.parametrize("H,Hkv,Sq", ROWS)
def test_rows_masks_splits(H, Hkv, Sq, n_splits, mask):
    check(2, H, Hkv, Sq, 1500, 128, "bf16", mask, n_splits, seed=H * 31 + Hkv * 7 + Sq)


@pytest.mark.parametrize("Sk", [1, 31, 32, 33, 127, 128, 129, 255, 700, 4097])
@pytest.mark.parametrize("D,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16"), (128, "f16")])
def test_ragged_key_counts(Sk, D, dtype):
    """Key counts that end inside a 32-key group, on its edge and past a tile."""
    check(1, 8, 2, 1, Sk, D, dtype, "none", None, seed=Sk + D)
    check(1, 4, 4, 3, Sk, D, dtype, "bottomright", 0, seed=Sk + D + 1)


@pytest.mark.parametrize("D", [80, 96, 112])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_padded_head_dims(D, dtype):
    check(2, 8, 2, 1, 2000, D, dtype, "none", None, seed=D)
    check(2, 4, 4, 2, 900, D, dtype, "bottomright", 0, seed=D + 1)


@pytest.mark.parametrize("n_splits", [1, 2, 7, 64, 1024])
def test_split_counts_with_empty_ranges(n_splits):
    """Up to 1024 ranges over 3000 keys (most of them empty): a range with no key
    writes LSE = -inf and weight 0."""
    check(1, 8, 2, 1, 3000, 128, "bf16", "none", n_splits, seed=n_splits)
    check(1, 4, 4, 2, 3000, 64, "f16", "bottomright", n_splits, seed=n_splits + 1)


def test_topleft_rows_that_see_few_keys():
    """Top-left mask with grouped heads: packed row r is query position r % Sq, which
    sees keys 0 .. r % Sq only: every later tile, and every split range after the
    first, sees nothing of the row."""
    check(3, 8, 2, 4, 5000, 128, "bf16", "topleft", 0, seed=5)
    check(3, 8, 2, 4, 5000, 64, "f16", "topleft", 5, seed=6)


@pytest.mark.parametrize("scale", [-0.3, 0.0, 0.9])
@pytest.mark.parametrize("mask", ["none", "bottomright"])
def test_scales(scale, mask):
    """Negative and zero scales; 0.9 at D = 128 (scores of tens of log2 units, near
    one-hot rows, rescales of the running max)."""
    check(2, 8, 4, 1, 3000, 128, "bf16", mask, None, seed=11, scale=scale)
    check(2, 4, 4, 2, 3000, 64, "f16", mask, 0, seed=12, scale=scale)


def test_rising_keys_rescale():
    """K scaled by 3 and keys whose scores rise along the sequence: the running max of
    both warpgroups moves up tile after tile (the lazy rescale of O in tensor memory)."""
    B, H, Hkv, Sq, Sk, D = 1, 8, 2, 1, 4000, 128
    q, k, v = make_gqa(B, H, Hkv, Sq, Sk, D, "bf16", 13, k_scale=3.0)
    ramp = torch.linspace(0.0, 4.0, Sk).reshape(1, 1, Sk, 1)
    k = (k.float() + ramp * q.float()[:, :1, :1, :].sign()).to(torch.bfloat16)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=af.ATTN_MASK_NONE, scale=1 / np.sqrt(D))
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), af.ATTN_MASK_NONE, 1 / np.sqrt(D))
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= O_TOL
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= LSE_TOL


def test_whole_and_split_agree_and_repeat():
    """The same decode inputs through the whole pass twice (bit-identical) and through
    two split counts (equal within the tolerance)."""
    q, k, v = (t.cuda() for t in make_gqa(4, 16, 4, 1, 6000, 128, "bf16", 17))
    o1, l1 = af.attention_ex(q, k, v, n_splits=0)
    o2, l2 = af.attention_ex(q, k, v, n_splits=0)
    o3, l3 = af.attention_ex(q, k, v, n_splits=5)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert (o1.float() - o3.float()).abs().max().item() <= O_TOL
    assert (l1 - l3).abs().max().item() <= LSE_TOL
