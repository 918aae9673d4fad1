"""GEMM with the fused bias + activation epilogue (gemm_bias_act, through the C ABI)
vs the fp64 oracle, element by element.

Tolerance, from the arithmetic: 16-bit products are exact in fp32 and accumulate in
fp32 on the tensor cores, so the pre-activation error is at most about
2^-18 * (sum_k |a_mk w_nk| + |bias_n|) (a generous bound on fp32 accumulation over
K <= 8192 terms); GELU's slope is below 1.13 and ReLU's is 1; the fp32 activation
adds ~2^-21 |C|; C is rounded once (half an ulp: 2^-11 fp16, 2^-8 bf16, relative).
So |C - C_ref| <= half_ulp |C_ref| + 1.13 * 2^-18 * (sum_k |a w| + |bias|) + 2^-24."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from workloads import GEMM_WORKLOADS, make_gemm

pytestmark = pytest.mark.gpu

HALF_ULP = {"f16": 2.0 ** -11, "bf16": 2.0 ** -8}
ACTS = {"none": af.GEMM_ACT_NONE, "gelu": af.GEMM_ACT_GELU, "relu": af.GEMM_ACT_RELU}


def check(c, a, w, b, act, dtype, what, rows=None):
    ad, wd = a.double().numpy(), w.double().numpy()
    bd = b.double().numpy() if b is not None else None
    if rows is not None:
        ad = ad[rows]
    ref = oracle.gemm_bias_act_ref(ad, wd, bd, act)
    mag = np.abs(ad) @ np.abs(wd).T + (np.abs(bd)[None, :] if bd is not None else 0.0)
    c = c.double().cpu().numpy()
    if rows is not None:
        c = c[rows]
    bound = HALF_ULP[dtype] * np.abs(ref) + 1.13 * 2.0 ** -18 * mag + 2.0 ** -24
    err = np.abs(c - ref)
    assert np.isfinite(c).all(), what
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), (f"{what}: worst {worst} c={c[worst]!r} ref={ref[worst]!r} "
                                  f"err={err[worst]:.3e} bound={bound[worst]:.3e}")


SHAPES = [(1, 8, 8), (128, 256, 64), (129, 264, 72), (300, 520, 1000), (1000, 8, 4096),
          (257, 1024, 200), (64, 2048, 8), (513, 777 // 8 * 8, 136), (2048, 512, 1024)]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("act", ["none", "gelu", "relu"])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_shapes(M, N, K, act, dtype):
    """Tile-aligned and ragged M (128-row tiles), N (256-column tiles) and K (64-wide
    blocks, K a multiple of 8), with a bias."""
    a, w, b = make_gemm(M, N, K, dtype, seed=M * 7 + N * 3 + K)
    c = af.gemm_bias_act(a.cuda(), w.cuda(), b.cuda(), ACTS[act])
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    check(c, a, w, b, ACTS[act], dtype, f"{M}x{N}x{K} {act} {dtype}")


@pytest.mark.parametrize("act", ["none", "gelu"])
def test_without_bias(act):
    a, w, _ = make_gemm(333, 768, 520, "bf16", seed=5)
    c = af.gemm_bias_act(a.cuda(), w.cuda(), None, ACTS[act])
    torch.cuda.synchronize()
    check(c, a, w, None, ACTS[act], "bf16", f"no bias {act}")


def test_many_tiles_per_cta_and_determinism():
    """More tiles than SMs (each CTA walks several, alternating accumulators); two runs
    are bit-identical."""
    a, w, b = make_gemm(2048, 4096, 256, "f16", seed=8)
    da, dw, db = a.cuda(), w.cuda(), b.cuda()
    c1 = af.gemm_bias_act(da, dw, db, af.GEMM_ACT_GELU)
    c2 = af.gemm_bias_act(da, dw, db, af.GEMM_ACT_GELU)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    rows = np.arange(0, 2048, 37)
    check(c1, a, w, b, af.GEMM_ACT_GELU, "f16", "many tiles", rows=rows)


def test_timeout_is_reported_and_the_context_survives():
    """Debug flag 1: the producer loads nothing, the MMA warp's first wait runs out
    after 2 s, the kernel ends with ATTN_ERR_TIMEOUT in the status word; a normal call
    right after still matches the oracle."""
    a, w, b = make_gemm(256, 512, 128, "bf16", seed=9)
    da, dw, db = a.cuda(), w.cuda(), b.cuda()
    c = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
    rc = af.gemm_bias_act_raw(da.data_ptr(), dw.data_ptr(), db.data_ptr(), c.data_ptr(), 256,
                              512, 128, af.GEMM_ACT_NONE, af.ATTN_BF16,
                              torch.cuda.current_stream().cuda_stream, flags=1)
    assert rc == af.ATTN_OK
    assert af.attn_fwd_status() == af.ATTN_ERR_TIMEOUT
    assert af.attn_fwd_status() == 0
    # the same with the 256-row tiles (flag 4)
    rc = af.gemm_bias_act_raw(da.data_ptr(), dw.data_ptr(), db.data_ptr(), c.data_ptr(), 256,
                              512, 128, af.GEMM_ACT_NONE, af.ATTN_BF16,
                              torch.cuda.current_stream().cuda_stream, flags=1 | 4)
    assert rc == af.ATTN_OK
    assert af.attn_fwd_status() == af.ATTN_ERR_TIMEOUT
    c = af.gemm_bias_act(da, dw, db, af.GEMM_ACT_NONE)
    torch.cuda.synchronize()
    check(c, a, w, b, af.GEMM_ACT_NONE, "bf16", "after timeout")


@pytest.mark.parametrize("name", list(GEMM_WORKLOADS))
def test_benchmark_workloads_sampled_rows(name):
    """The benchmark's GEMM workloads at full size: sampled rows (first, last, every
    128-row tile boundary of the first 8 tiles, random) of C against the oracle."""
    g = GEMM_WORKLOADS[name]
    a, w, b = make_gemm(g.M, g.N, g.K, g.dtype, g.seed)
    c = af.gemm_bias_act(a.cuda(), w.cuda(), b.cuda(), g.act)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    assert torch.isfinite(c.float()).all()
    rng = np.random.default_rng(g.seed)
    rows = np.unique(np.concatenate([[0, g.M - 1], np.arange(127, 1024, 128),
                                     np.arange(128, 1024, 128), rng.choice(g.M, 8)]))
    check(c, a, w, b, g.act, g.dtype, name, rows=rows)


@pytest.mark.parametrize("tiles", [2, 4])
@pytest.mark.parametrize("M,N,K", [(257, 264, 2048), (1000, 512, 64), (128, 1024, 4096),
                                   (384, 256, 136)])
def test_both_tile_shapes(M, N, K, tiles):
    """Debug flag 2 / 4 forces the 128-row / 256-row output tiles: both give the oracle's
    result on tile-aligned and ragged shapes (the default picks by K)."""
    a, w, b = make_gemm(M, N, K, "bf16", seed=M + N + K + tiles)
    da, dw, db = a.cuda(), w.cuda(), b.cuda()
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rc = af.gemm_bias_act_raw(da.data_ptr(), dw.data_ptr(), db.data_ptr(), c.data_ptr(), M, N,
                              K, af.GEMM_ACT_GELU, af.ATTN_BF16,
                              torch.cuda.current_stream().cuda_stream, flags=tiles)
    assert rc == af.ATTN_OK
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    check(c, a, w, b, af.GEMM_ACT_GELU, "bf16", f"{M}x{N}x{K} tiles flag {tiles}")


def test_bias_not_16_byte_aligned():
    """A bias that starts 2 bytes past a 16-byte boundary takes the element-wise bias
    loads; the result is the same."""
    M, N, K = 300, 264, 200
    a, w, b = make_gemm(M, N, K, "f16", seed=77)
    da, dw = a.cuda(), w.cuda()
    store = torch.zeros(N + 8, dtype=torch.float16, device="cuda")
    store[1:N + 1] = b.cuda()
    db = store[1:N + 1]
    assert db.data_ptr() % 16 == 2
    c = torch.empty((M, N), dtype=torch.float16, device="cuda")
    rc = af.gemm_bias_act_raw(da.data_ptr(), dw.data_ptr(), db.data_ptr(), c.data_ptr(), M, N,
                              K, af.GEMM_ACT_GELU, af.ATTN_F16,
                              torch.cuda.current_stream().cuda_stream)
    assert rc == af.ATTN_OK
    torch.cuda.synchronize()
    check(c, a, w, b, af.GEMM_ACT_GELU, "f16", "unaligned bias")
    c2 = af.gemm_bias_act(da, dw, b.cuda(), af.GEMM_ACT_GELU)
    torch.cuda.synchronize()
    assert torch.equal(c, c2)
