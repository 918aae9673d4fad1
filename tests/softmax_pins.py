"""Pins for the fp64 row-softmax oracle: facts that do not come from the oracle.

Each pin is a function of the loaded oracle library, so the same checks run against
deliberately broken copies (tests/test_softmax_oracle.py).  The facts come from the
mathematics of the softmax (the operation of the tutorial's fused-softmax step,
pro.edgex.exchange summary, fused-softmax paragraph):
  * closed forms: a constant row is uniform (1/n); a two-element row [a, b] gives
    1 / (1 + e^(b - a)); a row with one entry far above the rest is one-hot;
  * invariants: rows sum to one, adding a constant to a row changes nothing,
    permuting a row permutes its output;
  * a library routine the definition reduces to: torch.softmax in float64 on the CPU.
"""
import math

import numpy as np
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def spin_constant_row(lib):
    for n in (1, 2, 7, 1000):
        y = oracle.softmax_ref(np.full((3, n), 2.5), lib=lib)
        np.testing.assert_allclose(y, 1.0 / n, rtol=1e-15, atol=0)


def spin_two_elements(lib):
    a, b = 0.3, -1.7
    y = oracle.softmax_ref(np.array([[a, b], [b, a]]), lib=lib)
    p = 1.0 / (1.0 + math.exp(b - a))
    np.testing.assert_allclose(y, [[p, 1 - p], [1 - p, p]], rtol=1e-15, atol=1e-16)


def spin_huge_margin_one_hot(lib):
    """Entries near +-1e4 would overflow exp without the max subtraction."""
    x = _rand((4, 50), 1)
    hot = [3, 0, 49, 17]
    for r, j in enumerate(hot):
        x[r, j] = 1.0e4
    x[1] -= 2.0e4                       # a row of large negative values
    x[1, hot[1]] = -1.0e4
    y = oracle.softmax_ref(x, lib=lib)
    expect = np.zeros_like(x)
    expect[np.arange(4), hot] = 1.0
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-300)


def spin_rows_sum_to_one_and_shift(lib):
    x = _rand((16, 333), 2, 3.0)
    y = oracle.softmax_ref(x, lib=lib)
    assert (y > 0).all()
    np.testing.assert_allclose(y.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    c = _rand((16, 1), 3, 50.0)
    np.testing.assert_allclose(oracle.softmax_ref(x + c, lib=lib), y, rtol=1e-12, atol=0)


def spin_permutation(lib):
    x = _rand((5, 64), 4, 2.0)
    perm = np.random.default_rng(5).permutation(64)
    y = oracle.softmax_ref(x, lib=lib)
    np.testing.assert_allclose(oracle.softmax_ref(x[:, perm], lib=lib), y[:, perm],
                               rtol=1e-14, atol=0)


def spin_torch_softmax(lib):
    for (rows, n, seed, s) in ((7, 1, 6, 1.0), (9, 129, 7, 4.0), (3, 5000, 8, 10.0)):
        x = _rand((rows, n), seed, s)
        ref = torch.softmax(torch.from_numpy(x), dim=-1).numpy()
        np.testing.assert_allclose(oracle.softmax_ref(x, lib=lib), ref, rtol=1e-13, atol=1e-300)


ALL_SOFTMAX_PINS = [spin_constant_row, spin_two_elements, spin_huge_margin_one_hot,
                    spin_rows_sum_to_one_and_shift, spin_permutation, spin_torch_softmax]
