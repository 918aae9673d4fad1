"""The standalone row softmax (row_softmax, through the C ABI) vs the fp64 oracle,
element by element.

Tolerance, from the arithmetic: the kernel computes exp of d = x - max in fp32 (ex2 of
d*log2(e), relative error about 2^-22), sums in fp32 and rounds y once to its dtype.
So |y - y_ref| <= (half an ulp of the output type + 2^-24 * (64 + n / 64)) * y_ref
+ the smallest step of the output type near zero (2^-25 for fp16 subnormals; 2^-126
for bf16 / fp32, whose exp flushes results below it to zero).  The n-dependent term
bounds the fp32 sum (at most ~n/1024 sequential additions per thread plus a tree)."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from workloads import SOFTMAX_WORKLOADS, make_rows

pytestmark = pytest.mark.gpu

HALF_ULP = {"f16": 2.0 ** -11, "bf16": 2.0 ** -8, "f32": 2.0 ** -24}
ABS = {"f16": 2.0 ** -25, "bf16": 2.0 ** -126, "f32": 2.0 ** -126}


def check(y, x_cpu, dtype, what):
    y = y.double().cpu().numpy()
    ref = oracle.softmax_ref(x_cpu.double().numpy())
    n = ref.shape[-1]
    rel = HALF_ULP[dtype] + 2.0 ** -24 * (64 + n / 64)
    err = np.abs(y - ref)
    bound = rel * np.abs(ref) + ABS[dtype]
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.isfinite(y).all(), what
    assert (err <= bound).all(), (f"{what}: worst {worst} y={y[worst]!r} ref={ref[worst]!r} "
                                  f"err={err[worst]:.3e} bound={bound[worst]:.3e}")


SHAPES = [(1, 1), (3, 7), (5, 8), (64, 100), (33, 1000), (16, 1024), (8, 4096), (4, 4097),
          (4, 8192), (3, 30000), (2, 65536), (2, 65537), (2, 131072), (1, 1 << 20),
          (10000, 512), (7, 2048), (9, 3000)]


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("rows,n", SHAPES)
def test_shapes(rows, n, dtype):
    """Every dispatch path: a warp per row (rows up to 8 KB), a CTA per row (to
    128 KB), two passes (longer rows, or lengths that break 16-byte alignment)."""
    x = make_rows(rows, n, dtype, seed=rows * 31 + n, scale=4.0)
    y = af.row_softmax(x.cuda())
    torch.cuda.synchronize()
    check(y, x, dtype, f"{rows}x{n} {dtype}")


@pytest.mark.parametrize("dtype,big", [("f16", 60000.0), ("bf16", 1e30), ("f32", 1e30)])
def test_large_magnitudes_need_the_max_subtraction(dtype, big):
    """Rows of huge positive or negative values (exp would overflow or underflow
    without subtracting the row max), one hot entry per row, some ties."""
    for n in (100, 4096, 40000):
        x = make_rows(6, n, "f32", seed=n, scale=1.0)
        x[0] += big * 0.5
        x[1] -= big * 0.9
        x[2, 7] = big
        x[3, :] = -big
        x[4, ::3] = big
        x = x.to({"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[dtype])
        y = af.row_softmax(x.cuda())
        torch.cuda.synchronize()
        check(y, x, dtype, f"big {dtype} n={n}")


@pytest.mark.parametrize("n", [1000, 4096, 50000, 300000])
def test_in_place_equals_out_of_place(n):
    x = make_rows(5, n, "bf16", seed=3, scale=3.0).cuda()
    y = af.row_softmax(x)
    x2 = x.clone()
    af.row_softmax(x2, out=x2)
    torch.cuda.synchronize()
    assert torch.equal(x2, y)


def test_no_rows_is_a_no_op():
    x = torch.empty((0, 128), dtype=torch.float16, device="cuda")
    assert af.row_softmax(x).numel() == 0


@pytest.mark.parametrize("name", list(SOFTMAX_WORKLOADS))
def test_benchmark_workloads_sampled_rows(name):
    """The benchmark's row-softmax workloads at full size: sampled rows against the
    oracle; every row sums to one within the fp32 sum bound."""
    w = SOFTMAX_WORKLOADS[name]
    x = make_rows(w.rows, w.n, w.dtype, w.seed, w.scale)
    y = af.row_softmax(x.cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    sums = y.double().sum(dim=1).cpu().numpy()
    assert np.abs(sums - 1).max() <= HALF_ULP[w.dtype] * 4 + 2.0 ** -24 * (64 + w.n / 64) * 4
    rows = np.random.default_rng(w.seed).choice(w.rows, size=min(32, w.rows), replace=False)
    rows = np.unique(np.concatenate([rows, [0, w.rows - 1]]))
    idx = torch.from_numpy(rows)
    check(y[idx.cuda()], x[idx], w.dtype, name)
