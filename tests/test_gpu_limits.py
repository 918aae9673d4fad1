"""The size limits of the C ABI, at their edges, against the fp64 oracle (sampled rows):
sequences of 2^24 - 1 keys or queries (offsets past 2^31 elements in K/V or Q/O), 2^24
heads, and a 2^24-key decode through the split pass.  Each case holds a few GB on the
device."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import compare

pytestmark = pytest.mark.gpu

MAX = (1 << 24) - 1


def randn16(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(dtype)


def test_longest_key_sequence_whole_and_split():
    """One query row per head against 2^24 - 1 keys (K, V 4 GB each): the last KV tile
    is ragged and element offsets exceed 2^31."""
    B, H, Sq, Sk, D = 1, 1, 1, MAX, 128
    q, k, v = randn16((B, H, Sq, D), 1), randn16((B, H, Sk, D), 2), randn16((B, H, Sk, D), 3)
    scale = 0.09
    o_w, l_w = af.attention(q, k, v, scale=scale)
    o_s, l_s = af.attention_ex(q, k, v, scale=scale, n_splits=None)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    ro, rl = oracle.attn_ref_rows(q.double().cpu().numpy(), k.double().cpu().numpy(),
                                  v.double().cpu().numpy(), [(0, 0, 0)], False, scale)
    for o, l, what in ((o_w, l_w, "whole"), (o_s, l_s, "split")):
        compare(o.double().cpu().numpy()[0, 0], l.double().cpu().numpy()[0, 0], ro, rl, what)


def test_longest_query_sequence_causal():
    """2^24 - 1 query rows (Q, O 4 GB each) against 300 keys, causal: rows past the
    keys see them all; first, ragged-tail and last rows against the oracle."""
    B, H, Sq, Sk, D = 1, 1, MAX, 300, 128
    q, k, v = randn16((B, H, Sq, D), 4), randn16((B, H, Sk, D), 5), randn16((B, H, Sk, D), 6)
    o, lse = af.attention(q, k, v, causal=True, scale=0.1)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    rows = [(0, 0, i) for i in (0, 1, 127, 128, 299, 300, 1 << 20, MAX - 128, MAX - 1)]
    idx = torch.tensor([r[2] for r in rows], device="cuda")
    ro, rl = _oracle_rows(q, k, v, rows, 0.1)
    compare(o[0, 0, idx].double().cpu().numpy(), lse[0, 0, idx].double().cpu().numpy(), ro, rl,
            "longest query sequence")


def _oracle_rows(q, k, v, rows, scale):
    """Oracle rows of a causal pass without copying all of Q to the host: each sampled
    row i sees keys 0..min(i, Sk - 1), so it equals the non-causal oracle of that one
    query row against the first min(i + 1, Sk) keys."""
    Sk = k.shape[2]
    kd, vd = k.double().cpu().numpy(), v.double().cpu().numpy()
    outs, lses = [], []
    for (b, h, i) in rows:
        n = min(i + 1, Sk)
        qi = q[b:b + 1, h:h + 1, i:i + 1, :].double().cpu().numpy()
        o, l = oracle.attn_ref(qi, kd[b:b + 1, h:h + 1, :n], vd[b:b + 1, h:h + 1, :n], False,
                               scale)
        outs.append(o[0, 0, 0])
        lses.append(l[0, 0, 0])
    return np.array(outs), np.array(lses)


def test_most_heads():
    """B * H = 2^24 heads of 2 rows x 3 keys, D = 64 (2^24 units over the persistent
    grid): sampled heads against the oracle."""
    B, H, S, D = 1 << 12, 1 << 12, 2, 64
    q, k, v = (randn16((B, H, S, D), s, torch.float16) for s in (7, 8, 9))
    o, lse = af.attention(q, k, v, scale=0.125)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    rng = np.random.default_rng(0)
    for (b, h) in [(0, 0), (B - 1, H - 1)] + [tuple(x) for x in rng.integers(0, 1 << 12, (6, 2))]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        o_ref, l_ref = oracle.attn_ref(q[sl].double().cpu().numpy(), k[sl].double().cpu().numpy(),
                                       v[sl].double().cpu().numpy(), False, 0.125)
        compare(o[sl].double().cpu().numpy(), lse[sl].double().cpu().numpy(), o_ref, l_ref,
                f"head {b},{h}")


def test_over_the_limits_are_rejected():
    q = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    p = q.data_ptr()
    for (B, H, Sq, Sk) in ((1, 1, 1 << 24 | 1, 4), (1, 1, 4, 1 << 24 | 1), (1 << 12, 1 << 12 | 1, 1, 1)):
        rc = af.attn_fwd(p, p + (1 << 36), p + (2 << 36), p + (3 << 36), None, B, H, Sq, Sk, 128,
                         0, 0.1, af.ATTN_BF16, None)
        assert rc == af.ATTN_ERR_SHAPE, (B, H, Sq, Sk)
