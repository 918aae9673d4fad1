"""Head dimensions 192 and 256 (the wide kernel: one 128-row query tile per CTA, 64-key
K/V tiles, two S buffers in tensor memory) against the fp64 oracle, element by element,
through the C ABI: whole and split pass, both causal alignments, grouped K/V heads,
ragged and degenerate sizes, scales that force the lazy O rescale, and CTAs that walk
several work units.  Tolerances as everywhere: max |dO| <= 2e-2, max |dLSE| <= 1e-3."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import LSE_TOL, O_TOL
from workloads import make_qkv, sample_rows

pytestmark = pytest.mark.gpu

MASKS = {"none": af.ATTN_MASK_NONE, "topleft": af.ATTN_MASK_CAUSAL,
         "bottomright": af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT}
WIDE = [(192, "bf16"), (192, "f16"), (256, "bf16"), (256, "f16")]


def make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed):
    q, _, _ = make_qkv(B, H, Sq, 1, D, dtype, seed)
    _, k, v = make_qkv(B, Hkv, 1, Sk, D, dtype, seed + 100003)
    return q, k, v


def compare(o, lse, o_ref, lse_ref, what):
    assert np.isfinite(o).all(), what
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: empty rows differ"
    assert (o[empty] == 0).all(), f"{what}: O of an empty row is not 0"
    do = np.abs(o - o_ref).max()
    dl = np.abs(lse[~empty] - lse_ref[~empty]).max() if (~empty).any() else 0.0
    assert do <= O_TOL and dl <= LSE_TOL, f"{what}: max dO {do:.3e} max dLSE {dl:.3e}"


def run_and_check(q, k, v, mask, scale, n_splits, what):
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=MASKS[mask], scale=scale, n_splits=n_splits)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0, what
    o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), MASKS[mask], scale)
    compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, what)


def check(B, H, Hkv, Sq, Sk, D, dtype, mask, n_splits, seed, scale=None):
    q, k, v = make_gqa(B, H, Hkv, Sq, Sk, D, dtype, seed)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    run_and_check(q, k, v, mask, scale, n_splits,
                  f"B{B} H{H}/{Hkv} Sq{Sq} Sk{Sk} D{D} {dtype} {mask} n{n_splits} s{scale}")


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
@pytest.mark.parametrize("Sq,Sk", [(300, 500), (500, 500), (129, 257), (64, 1000),
                                   (400, 150)])
def test_whole_pass(Sq, Sk, mask, D, dtype):
    """Several 64-key tiles and 128-row query tiles with ragged tails; with the
    bottom-right mask and Sq > Sk the first rows see no key (O = 0, LSE = -inf)."""
    check(2, 3, 3, Sq, Sk, D, dtype, mask, 0, seed=Sq * 7 + Sk + D)


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("Sq,Sk", [(1, 1), (1, 65), (1, 64), (65, 1), (2, 3), (128, 64)])
def test_degenerate_sizes(Sq, Sk, D, dtype):
    for mask in ("none", "topleft", "bottomright"):
        check(1, 2, 2, Sq, Sk, D, dtype, mask, 0, seed=Sq + 3 * Sk)


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("n_splits", [None, 2, 3, 7, 40])
@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
def test_split_pass(mask, n_splits, D, dtype):
    """KV ranges of an odd number of 64-key tiles: causal rows of a query tile that see
    nothing of a range (partials O = 0, LSE = -inf) and ranges past every key."""
    check(1, 2, 2, 600, 600, D, dtype, mask, n_splits, seed=D + (n_splits or 0))


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("Sq,Sk", [(1, 5000), (4, 3000), (33, 2000)])
def test_split_decode_shapes(Sq, Sk, D, dtype):
    check(2, 4, 4, Sq, Sk, D, dtype, "none", None, seed=Sq + Sk)
    check(2, 4, 4, Sq, Sk, D, dtype, "bottomright", None, seed=Sq + Sk + 1)


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
@pytest.mark.parametrize("n_splits", [0, None, 5])
def test_grouped_heads(n_splits, mask, D, dtype):
    """8 query heads on 2 K/V heads: 4 x 40 packed rows per K/V head, query tiles that
    straddle query heads."""
    check(1, 8, 2, 40, 700, D, dtype, mask, n_splits, seed=D + 9)


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("scale", [-0.2, 0.0, "large"])
@pytest.mark.parametrize("mask", ["none", "topleft", "bottomright"])
@pytest.mark.parametrize("n_splits", [0, 3])
def test_unusual_scales(n_splits, mask, scale, D, dtype):
    """Negative and zero scales (their own instantiations) and a large one (scores with
    a spread of hundreds: the running max moves by more than 2^8 often).  The large
    scale is 1.0 in fp16 and 0.5 in bf16: a near one-hot softmax puts |O| close to
    max |v| (about 4.5 here), where bf16's own rounding of O (half an ulp, 1/64 in
    [4, 8)) plus that of P (up to 2^-9 relative, times |v|) can pass the 2e-2 bound."""
    if scale == "large":
        scale = 1.0 if dtype == "f16" else 0.5
    check(1, 2, 2, 300, 700, D, dtype, mask, n_splits, seed=int(scale * 10) + D, scale=scale)


@pytest.mark.parametrize("D,dtype", WIDE)
def test_rising_keys_force_rescales(D, dtype):
    """Keys whose norm grows along the sequence: the row max rises tile after tile, so
    O is rescaled on most tiles, each after the previous P V has finished."""
    q, k, v = make_qkv(1, 2, 200, 2048, D, dtype, seed=D + 77)
    ramp = (1.0 + torch.arange(2048, dtype=torch.float32) / 128.0).view(1, 1, -1, 1)
    k = (k.float() * ramp).to(k.dtype)
    for mask in ("none", "bottomright"):
        run_and_check(q, k, v, mask, 0.5 / np.sqrt(D), 0, f"rising keys D{D} {mask}")


@pytest.mark.parametrize("D,dtype", WIDE)
@pytest.mark.parametrize("mask", ["none", "topleft"])
def test_ctas_walk_several_units(mask, D, dtype):
    """160 units on at most 148 CTAs: the barrier phases run on across units."""
    check(2, 40, 40, 130, 200, D, dtype, mask, 0, seed=D + 123)
    check(1, 20, 20, 512, 512, D, dtype, mask, 0, seed=D + 124)


@pytest.mark.parametrize("D", [192, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_large_sampled_rows(causal, D):
    """B = 2, H = 16, Sq = Sk = 4096 in bf16 (the size the benchmark times), checked on
    sampled rows, tile boundaries included."""
    B, H, S = 2, 16, 4096
    q, k, v = make_qkv(B, H, S, S, D, "bf16", seed=D + int(causal))
    scale = 1.0 / np.sqrt(D)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention_ex(dq, dk, dv, mask=MASKS["topleft" if causal else "none"],
                             scale=scale, n_splits=0)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    rows = sample_rows(B, H, S, 48, seed=D)
    ro, rl = oracle.attn_ref_rows(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                  rows, causal, scale)
    idx = tuple(np.array(rows).T)
    compare(o.double().cpu().numpy()[idx], lse.double().cpu().numpy()[idx], ro, rl,
            f"D{D} causal={causal}")


def test_split_entry_points_and_workspace_size():
    """attn_fwd_splitkv (D = 256) equals attn_fwd_ex with the same split count, bit for
    bit, and the workspace formula holds for D = 192 and 256."""
    q, k, v = make_qkv(1, 4, 3, 3000, 256, "bf16", seed=5)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o1, l1 = af.attention_splitkv(dq, dk, dv, causal=False, scale=0.06, n_splits=6)
    o2, l2 = af.attention_ex(dq, dk, dv, mask=af.ATTN_MASK_NONE, scale=0.06, n_splits=6)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for D in (192, 256):
        o_bytes = (6 * 1 * 4 * 3 * D * 4 + 255) // 256 * 256
        assert af.splitkv_workspace_bytes(1, 4, 3, D, 6) == o_bytes + 6 * 4 * 3 * 4
