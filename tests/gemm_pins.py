"""Pins for the fp64 GEMM + bias + activation oracle: facts that do not come from the
oracle.

Each pin is a function of the loaded library, so the same checks run against
deliberately broken copies (tests/test_gemm_oracle.py).  The facts: identity and
permutation matrices (C = A or a column permutation of A), a rank-one case in closed
form, GELU at points where Phi is known (GELU(0) = 0, GELU(1) = Phi(1), GELU(-1) =
-Phi(-1), the odd part z - GELU(z) = GELU(-z)), ReLU by sign, the bias broadcast
along rows, and torch's float64 linear + gelu(approximate='none') / relu on random
shapes.
"""
import math

import numpy as np
import torch

import oracle

PHI1 = 0.5 * (1.0 + math.erf(1.0 / math.sqrt(2.0)))  # standard normal CDF at 1


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def gpin_identity_and_permutation(lib):
    a = _rand((5, 6), 1)
    c = oracle.gemm_bias_act_ref(a, np.eye(6), lib=lib)
    np.testing.assert_array_equal(c, a)
    perm = np.random.default_rng(2).permutation(6)
    c = oracle.gemm_bias_act_ref(a, np.eye(6)[perm], lib=lib)
    np.testing.assert_array_equal(c, a[:, perm])


def gpin_rank_one(lib):
    """A = u 1^T, W = v 1^T (K columns of ones): C[m,n] = K * u_m * v_n (exact in
    binary for small integers)."""
    u, v, K = np.arange(1, 4, dtype=float), np.arange(2, 7, dtype=float), 9
    c = oracle.gemm_bias_act_ref(np.outer(u, np.ones(K)), np.outer(v, np.ones(K)), lib=lib)
    np.testing.assert_array_equal(c, K * np.outer(u, v))


def gpin_bias_broadcast(lib):
    a, w, b = _rand((4, 3), 3), _rand((5, 3), 4), _rand((5,), 5)
    c0 = oracle.gemm_bias_act_ref(a, w, lib=lib)
    c = oracle.gemm_bias_act_ref(a, w, b, lib=lib)
    np.testing.assert_allclose(c - c0, np.broadcast_to(b, c.shape), rtol=0, atol=1e-14)


def gpin_gelu_points(lib):
    """With A = [[z]] and W = [[1]], C = GELU(z)."""
    def g(z):
        return oracle.gemm_bias_act_ref(np.array([[z]]), np.array([[1.0]]),
                                        act=oracle.ACT_GELU, lib=lib)[0, 0]
    assert g(0.0) == 0.0
    np.testing.assert_allclose(g(1.0), PHI1, rtol=1e-15)
    np.testing.assert_allclose(g(-1.0), -(1.0 - PHI1), rtol=1e-14)
    for z in (0.3, 1.7, 4.0, 9.0):
        np.testing.assert_allclose(z - g(z), -g(-z), rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(g(40.0), 40.0, rtol=1e-15)


def gpin_relu_sign(lib):
    a = _rand((6, 4), 6)
    w = np.eye(4)
    c = oracle.gemm_bias_act_ref(a, w, act=oracle.ACT_RELU, lib=lib)
    np.testing.assert_array_equal(c, np.where(a > 0, a, 0.0))


def gpin_torch_linear(lib):
    for (M, N, K, seed) in ((7, 9, 13, 10), (33, 17, 64, 11), (1, 1, 1, 12)):
        a, w, b = _rand((M, K), seed), _rand((N, K), seed + 1), _rand((N,), seed + 2)
        ta, tw, tb = (torch.from_numpy(x) for x in (a, w, b))
        z = torch.nn.functional.linear(ta, tw, tb)
        for act, ref in ((oracle.ACT_NONE, z),
                         (oracle.ACT_GELU, torch.nn.functional.gelu(z, approximate="none")),
                         (oracle.ACT_RELU, torch.relu(z))):
            c = oracle.gemm_bias_act_ref(a, w, b, act, lib=lib)
            np.testing.assert_allclose(c, ref.numpy(), rtol=1e-13, atol=1e-13)
        c = oracle.gemm_bias_act_ref(a, w, None, oracle.ACT_GELU, lib=lib)
        ref = torch.nn.functional.gelu(torch.nn.functional.linear(ta, tw), approximate="none")
        np.testing.assert_allclose(c, ref.numpy(), rtol=1e-13, atol=1e-13)


ALL_GEMM_PINS = [gpin_identity_and_permutation, gpin_rank_one, gpin_bias_broadcast,
                 gpin_gelu_points, gpin_relu_sign, gpin_torch_linear]
