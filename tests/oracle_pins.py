"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Every pin is a function of the loaded oracle library so the same checks can run
against deliberately broken copies of the oracle (tests/test_oracle_mutants.py):
a plausible mistake anywhere in the oracle -- a dropped scale, a wrong sign, a
mask on the wrong side or off by one, a wrong key or value index, a missing max
subtraction, a wrong log base -- must make at least one pin fail.

The facts come from the mathematics of softmax attention (the operation the
tutorial's fused FlashAttention forward must reproduce, pro.edgex.exchange summary,
FlashAttention paragraph), not from the oracle's code:
  * closed forms: one key; Q = 0 (uniform weights); constant V; causal row 0;
    one-hot attention with a huge margin; hand-worked 2x2 / 3x2 cases;
  * invariants: probability rows sum to one, masked weights are exactly zero,
    joint permutation of (K, V) rows, a common shift of every key, linearity in V;
  * a library routine the definition reduces to: PyTorch's float64 math-backend
    scaled_dot_product_attention on the CPU, and torch.logsumexp for the LSE.
"""
import math

import numpy as np
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape) * scale


def pin_single_key(lib):
    """Sk = 1: every query attends only to key 0, so O = V[0] and LSE = s_00."""
    B, H, Sq, D = 2, 3, 5, 7
    q, k, v = _rand((B, H, Sq, D), 1), _rand((B, H, 1, D), 2), _rand((B, H, 1, D), 3)
    for causal in (False, True):
        o, lse = oracle.attn_ref(q, k, v, causal, 0.37, lib=lib)
        np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-15)
        s = 0.37 * np.einsum("bhid,bhd->bhi", q, k[:, :, 0, :])
        np.testing.assert_allclose(lse, s, rtol=1e-14, atol=1e-14)


def pin_zero_query(lib):
    """Q = 0: all visible scores are equal, so O is the mean of the visible V rows
    and LSE = ln(number of visible keys).  Causal, top-left: row i sees keys 0..i."""
    B, H, Sq, Sk, D = 1, 2, 6, 9, 4
    q = np.zeros((B, H, Sq, D))
    k, v = _rand((B, H, Sk, D), 4), _rand((B, H, Sk, D), 5)
    o, lse = oracle.attn_ref(q, k, v, False, 0.5, lib=lib)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape),
                               rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.full(lse.shape, math.log(Sk)), rtol=0, atol=1e-14)
    o, lse = oracle.attn_ref(q, k, v, True, 0.5, lib=lib)
    for i in range(Sq):
        np.testing.assert_allclose(o[:, :, i, :], v[:, :, : i + 1, :].mean(axis=2),
                                   rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, i], math.log(i + 1), rtol=0, atol=1e-14)


def pin_constant_value(lib):
    """Every row of V equal to c: O = c whatever the weights."""
    B, H, Sq, Sk, D = 2, 2, 7, 11, 5
    q, k = _rand((B, H, Sq, D), 6, 2.0), _rand((B, H, Sk, D), 7, 2.0)
    c = _rand((D,), 8)
    v = np.broadcast_to(c, (B, H, Sk, D)).copy()
    for causal in (False, True):
        o, _ = oracle.attn_ref(q, k, v, causal, 0.9, lib=lib)
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13)


def pin_causal_first_row(lib):
    """Causal row 0 sees only key 0: O[0] = V[0], LSE[0] = scale * q_0 . k_0."""
    B, H, Sq, Sk, D = 2, 2, 8, 8, 6
    q, k, v = _rand((B, H, Sq, D), 9), _rand((B, H, Sk, D), 10), _rand((B, H, Sk, D), 11)
    o, lse = oracle.attn_ref(q, k, v, True, 0.25, lib=lib)
    np.testing.assert_allclose(o[:, :, 0, :], v[:, :, 0, :], rtol=0, atol=1e-15)
    s00 = 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0, :], k[:, :, 0, :])
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=1e-14, atol=1e-14)


def pin_hand_2x2(lib):
    """Hand-worked case, scale 1: Q = K = I (2x2), V = [[1,2],[3,4]].
    Non-causal row 0 has scores (1, 0): weights (e, 1)/(e+1); row 1 has (0, 1).
    Both LSEs are ln(1 + e).  Causal row 0 sees key 0 only: O = (1, 2), LSE = 1."""
    e = math.e
    q = np.eye(2).reshape(1, 1, 2, 2)
    k = np.eye(2).reshape(1, 1, 2, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 1, 2, 2)
    o, lse = oracle.attn_ref(q, k, v, False, 1.0, lib=lib)
    want = np.array([[(e * 1 + 3) / (e + 1), (e * 2 + 4) / (e + 1)],
                     [(1 + e * 3) / (e + 1), (2 + e * 4) / (e + 1)]])
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], [math.log1p(e)] * 2, rtol=1e-15, atol=1e-15)
    o, lse = oracle.attn_ref(q, k, v, True, 1.0, lib=lib)
    np.testing.assert_allclose(o[0, 0], [[1.0, 2.0], want[1]], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], [1.0, math.log1p(e)], rtol=1e-15, atol=1e-15)


def pin_hand_3x2_causal(lib):
    """Hand-worked Sq = 3 > Sk = 2, causal top-left, scale 1/2.
    q = (2, 0), (0, 2), (2, 2); k = (1, 0), (0, 1); V = [[1, -1], [5, 3]].
    Scaled scores: row 0 (1, 0), row 1 (0, 1), row 2 (1, 1).  Row 0 sees key 0 only;
    rows 1 and 2 see both keys (j <= i for every key)."""
    e = math.e
    q = np.array([[2.0, 0.0], [0.0, 2.0], [2.0, 2.0]]).reshape(1, 1, 3, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 1, 2, 2)
    v = np.array([[1.0, -1.0], [5.0, 3.0]]).reshape(1, 1, 2, 2)
    o, lse = oracle.attn_ref(q, k, v, True, 0.5, lib=lib)
    want_o = np.array([[1.0, -1.0],
                       [(1 + 5 * e) / (1 + e), (-1 + 3 * e) / (1 + e)],
                       [3.0, 1.0]])
    want_lse = np.array([1.0, math.log1p(e), 1.0 + math.log(2.0)])
    np.testing.assert_allclose(o[0, 0], want_o, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], want_lse, rtol=1e-15, atol=1e-15)


def pin_one_hot_huge_margin(lib):
    """Orthonormal keys and q_i = 1000 * k_t(i): score 1000 on key t, 0 elsewhere.
    Then O_i = V[t] (the other weights are e^-1000, below fp64 resolution) and
    LSE_i = 1000 + ln(1 + (Sk - 1) e^-1000) = 1000.  Without the max subtraction
    exp(1000) overflows, so this also pins the numerically safe softmax."""
    Sk = D = 8
    k = np.eye(D).reshape(1, 1, Sk, D)
    targets = [3, 0, 7, 5]
    q = np.stack([1000.0 * k[0, 0, t] for t in targets]).reshape(1, 1, len(targets), D)
    v = _rand((1, 1, Sk, D), 12)
    o, lse = oracle.attn_ref(q, k, v, False, 1.0, lib=lib)
    for r, t in enumerate(targets):
        np.testing.assert_allclose(o[0, 0, r], v[0, 0, t], rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[0, 0, r], 1000.0, rtol=1e-15, atol=0)


def pin_probability_rows(lib):
    """Probability rows are >= 0, sum to one, and are exactly 0 above the causal
    diagonal (top-left: j > i) and > 0 on and below it."""
    B, H, Sq, Sk, D = 1, 2, 9, 13, 4
    q, k, v = _rand((B, H, Sq, D), 13, 3.0), _rand((B, H, Sk, D), 14), _rand((B, H, Sk, D), 15)
    for causal in (False, True):
        _, _, p = oracle.attn_ref(q, k, v, causal, 0.5, return_probs=True, lib=lib)
        assert (p >= 0).all()
        np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-13)
        if causal:
            i = np.arange(Sq)[:, None]
            j = np.arange(Sk)[None, :]
            assert (p[..., j > i] == 0).all()
            assert (p[..., np.broadcast_to(j <= i, (Sq, Sk))] > 0).all()
        else:
            assert (p > 0).all()


def pin_permutation(lib):
    """Non-causal attention does not depend on the order of the (key, value) pairs."""
    B, H, Sq, Sk, D = 2, 1, 6, 10, 5
    q, k, v = _rand((B, H, Sq, D), 16), _rand((B, H, Sk, D), 17), _rand((B, H, Sk, D), 18)
    perm = np.random.default_rng(19).permutation(Sk)
    o1, l1 = oracle.attn_ref(q, k, v, False, 0.7, lib=lib)
    o2, l2 = oracle.attn_ref(q, k[:, :, perm], v[:, :, perm], False, 0.7, lib=lib)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)


def pin_key_shift(lib):
    """Adding one vector u to every key adds scale * q_i . u to every score of row i:
    the weights (so O) do not change and LSE_i grows by exactly that amount."""
    B, H, Sq, Sk, D = 1, 2, 7, 7, 6
    q, k, v = _rand((B, H, Sq, D), 20), _rand((B, H, Sk, D), 21), _rand((B, H, Sk, D), 22)
    u = _rand((D,), 23, 2.0)
    for causal in (False, True):
        o1, l1 = oracle.attn_ref(q, k, v, causal, 0.6, lib=lib)
        o2, l2 = oracle.attn_ref(q, k + u, v, causal, 0.6, lib=lib)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l2 - l1, 0.6 * np.einsum("bhid,d->bhi", q, u),
                                   rtol=0, atol=1e-12)


def pin_linear_in_value(lib):
    """O is linear in V for fixed Q, K."""
    B, H, Sq, Sk, D = 1, 1, 5, 8, 3
    q, k = _rand((B, H, Sq, D), 24), _rand((B, H, Sk, D), 25)
    v1, v2 = _rand((B, H, Sk, D), 26), _rand((B, H, Sk, D), 27)
    for causal in (False, True):
        a, _ = oracle.attn_ref(q, k, v1, causal, 0.8, lib=lib)
        b, _ = oracle.attn_ref(q, k, v2, causal, 0.8, lib=lib)
        c, _ = oracle.attn_ref(q, k, 2.0 * v1 - 3.0 * v2, causal, 0.8, lib=lib)
        np.testing.assert_allclose(c, 2.0 * a - 3.0 * b, rtol=0, atol=1e-12)


def pin_torch_sdpa(lib):
    """PyTorch's float64 math SDPA on the CPU (is_causal is top-left aligned) and
    torch.logsumexp of the masked scaled scores, on random sizes incl. Sq != Sk."""
    rng = np.random.default_rng(28)
    for trial in range(6):
        B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
        Sq, Sk = int(rng.integers(1, 70)), int(rng.integers(1, 70))
        D = int(rng.choice([1, 3, 16, 64]))
        scale = float(rng.uniform(0.05, 1.5))
        q = torch.from_numpy(_rand((B, H, Sq, D), 100 + trial))
        k = torch.from_numpy(_rand((B, H, Sk, D), 200 + trial, 2.0))
        v = torch.from_numpy(_rand((B, H, Sk, D), 300 + trial))
        for causal in (False, True):
            o, lse = oracle.attn_ref(q.numpy(), k.numpy(), v.numpy(), causal, scale, lib=lib)
            with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
                ref = torch.nn.functional.scaled_dot_product_attention(
                    q, k, v, is_causal=causal, scale=scale)
            np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
            s = scale * (q @ k.transpose(-1, -2))
            if causal:
                keep = torch.ones(Sq, Sk, dtype=torch.bool).tril()
                s = s.masked_fill(~keep, float("-inf"))
            np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(),
                                       rtol=0, atol=1e-12)


def pin_rows_match_whole(lib):
    """The row entry point gives the whole entry point's rows, bit for bit."""
    B, H, Sq, Sk, D = 2, 3, 17, 23, 8
    q, k, v = _rand((B, H, Sq, D), 29), _rand((B, H, Sk, D), 30), _rand((B, H, Sk, D), 31)
    rows = [(0, 0, 0), (1, 2, 16), (0, 1, 5), (1, 0, 11)]
    for causal in (False, True):
        o, lse = oracle.attn_ref(q, k, v, causal, 0.3, lib=lib)
        ro, rl = oracle.attn_ref_rows(q, k, v, rows, causal, 0.3, lib=lib)
        for n, (b, h, i) in enumerate(rows):
            assert np.array_equal(ro[n], o[b, h, i])
            assert rl[n] == lse[b, h, i]


def pin_bottom_right_closed_forms(lib):
    """Bottom-right causal mask: query i sees keys 0 .. i + Sk - Sq.  With Q = 0 the
    visible weights are uniform, so O is the mean of those V rows and LSE = ln(count);
    with Sq > Sk the first Sq - Sk rows see nothing: O = 0, LSE = -inf (empty sum);
    with Sq = Sk it is the top-left mask (row i sees 0..i)."""
    for (Sq, Sk) in ((5, 9), (7, 3), (6, 6)):
        B, H, D = 1, 2, 4
        q = np.zeros((B, H, Sq, D))
        k, v = _rand((B, H, Sk, D), 40 + Sq), _rand((B, H, Sk, D), 50 + Sk)
        o, lse = oracle.attn_ref_ex(q, k, v, oracle.CAUSAL_BOTTOM_RIGHT, 0.5, lib=lib)
        for i in range(Sq):
            last = i + Sk - Sq          # last visible key
            if last < 0:
                assert (o[:, :, i, :] == 0.0).all()
                assert (lse[:, :, i] == -np.inf).all()
            else:
                np.testing.assert_allclose(o[:, :, i, :], v[:, :, : last + 1, :].mean(axis=2),
                                           rtol=0, atol=1e-14)
                np.testing.assert_allclose(lse[:, :, i], math.log(last + 1), rtol=0, atol=1e-14)


def pin_bottom_right_torch(lib):
    """PyTorch's float64 math SDPA with an explicit lower-right boolean mask
    (torch.tril with diagonal Sk - Sq) and torch.logsumexp of the masked scores;
    Sq <= Sk so no row is empty."""
    for (Sq, Sk, seed) in ((3, 11, 60), (17, 40, 61), (9, 9, 62)):
        B, H, D = 2, 3, 8
        q, k, v = _rand((B, H, Sq, D), seed), _rand((B, H, Sk, D), seed + 1), _rand((B, H, Sk, D), seed + 2)
        scale = 0.3
        o, lse = oracle.attn_ref_ex(q, k, v, oracle.CAUSAL_BOTTOM_RIGHT, scale, lib=lib)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        allowed = torch.tril(torch.ones(Sq, Sk, dtype=torch.bool), diagonal=Sk - Sq)
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed,
                                                                   scale=scale)
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        s = scale * torch.einsum("bhid,bhjd->bhij", tq, tk)
        s = s.masked_fill(~allowed, float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_grouped_heads_torch(lib):
    """K/V with fewer heads than Q: PyTorch's SDPA with enable_gqa (query head h reads
    K/V head h // (H // Hkv)), and the LSE of K expanded with repeat_interleave."""
    B, H, Hkv, Sq, Sk, D = 2, 8, 2, 6, 13, 8
    q, k, v = _rand((B, H, Sq, D), 70), _rand((B, Hkv, Sk, D), 71), _rand((B, Hkv, Sk, D), 72)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    for causal in (False, True):
        o, lse = oracle.attn_ref_ex(q, k, v, None, 0.4, causal=causal, lib=lib)
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
            ref = torch.nn.functional.scaled_dot_product_attention(
                tq, tk, tv, is_causal=causal, scale=0.4, enable_gqa=True)
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        ke = tk.repeat_interleave(H // Hkv, dim=1)
        s = 0.4 * torch.einsum("bhid,bhjd->bhij", tq, ke)
        if causal:
            s = s.masked_fill(~torch.tril(torch.ones(Sq, Sk, dtype=torch.bool)), float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)
    # the row entry point follows the same head mapping and mask
    rows = [(0, 7, 5), (1, 3, 0), (1, 4, 2)]
    for mask in (oracle.NO_MASK, oracle.CAUSAL_TOP_LEFT, oracle.CAUSAL_BOTTOM_RIGHT):
        o, lse = oracle.attn_ref_ex(q, k, v, mask, 0.4, lib=lib)
        ro, rl = oracle.attn_ref_rows_ex(q, k, v, rows, mask, 0.4, lib=lib)
        idx = tuple(np.array(rows).T)
        assert np.array_equal(ro, o[idx]) and np.array_equal(rl, lse[idx])


def pin_product_head_dims(lib):
    """PyTorch's float64 math SDPA at every head dimension the CUDA path accepts (64, 80,
    96, 112, 128, 192, 256), all three masks, Sq < Sk and Sq > Sk."""
    for n, D in enumerate((64, 80, 96, 112, 128, 192, 256)):
        for (Sq, Sk) in ((5, 9), (9, 4)):
            q = _rand((1, 2, Sq, D), 80 + n)
            k = _rand((1, 2, Sk, D), 90 + n)
            v = _rand((1, 2, Sk, D), 100 + n)
            scale = 1.0 / math.sqrt(D)
            tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
            masks = ((oracle.NO_MASK, torch.ones(Sq, Sk, dtype=torch.bool)),
                     (oracle.CAUSAL_TOP_LEFT, torch.ones(Sq, Sk, dtype=torch.bool).tril()),
                     (oracle.CAUSAL_BOTTOM_RIGHT,
                      torch.tril(torch.ones(Sq, Sk, dtype=torch.bool), diagonal=Sk - Sq)))
            for mask, allowed in masks:
                o, lse = oracle.attn_ref_ex(q, k, v, mask, scale, lib=lib)
                s = scale * torch.einsum("bhid,bhjd->bhij", tq, tk)
                s = s.masked_fill(~allowed, float("-inf"))
                np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(),
                                           rtol=0, atol=1e-12)
                seen = allowed.any(dim=1)   # rows with at least one visible key
                with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
                    ref = torch.nn.functional.scaled_dot_product_attention(
                        tq[:, :, seen], tk, tv, attn_mask=allowed[seen], scale=scale)
                np.testing.assert_allclose(o[:, :, seen.numpy()], ref.numpy(), rtol=0, atol=1e-12)
                assert (o[:, :, ~seen.numpy()] == 0.0).all()


ALL_PINS = [pin_single_key, pin_zero_query, pin_constant_value, pin_causal_first_row,
            pin_hand_2x2, pin_hand_3x2_causal, pin_one_hot_huge_margin,
            pin_probability_rows, pin_permutation, pin_key_shift, pin_linear_in_value,
            pin_torch_sdpa, pin_rows_match_whole,
            pin_bottom_right_closed_forms, pin_bottom_right_torch, pin_grouped_heads_torch,
            pin_product_head_dims]
