"""Fit the polynomial the attention kernel uses to compute 2^f on the FMA pipe.

Method: Cody-Waite style range reduction, 2^x = 2^n * 2^f with n = round(x) and
f = x - n in [-1/2, 1/2], then a polynomial P(f) ~ 2^f of degree `deg` whose maximum
*relative* error over [-1/2, 1/2] is minimised with the Remez exchange algorithm
(equioscillation of the weighted error (P(f) - 2^f) / 2^f at deg + 2 points).
The coefficients are then rounded to fp32 and the error of the fp32 evaluation
(Horner form, one fused multiply-add per step) is measured on a dense grid in
float64 arithmetic that mimics fp32 fma rounding.

    python fit_exp2_poly.py [deg]        prints the coefficients as C literals
"""
import sys

import numpy as np

LO, HI = -0.5, 0.5


def _target(x):
    return np.exp2(x)


def remez(deg, iters=30):
    n = deg + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    x = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve P(x_i) - 2^x_i = (-1)^i E 2^x_i for the deg+1 coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * _target(x[i])
        sol = np.linalg.solve(A, _target(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - _target(grid)) / _target(grid)
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sign[i] != sign[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return c, float(np.max(np.abs(err)))


def fp32_eval_error(c32):
    """Max relative error of the fp32 Horner evaluation with fused multiply-adds."""
    f = np.linspace(LO, HI, 400001).astype(np.float32).astype(np.float64)
    p = np.float64(c32[-1])
    for ck in c32[-2::-1]:
        # fma(p, f, ck) in fp32: exact product and sum in fp64, one rounding to fp32
        p = (p * f + np.float64(ck)).astype(np.float32).astype(np.float64)
    return float(np.max(np.abs(p - np.exp2(f)) / np.exp2(f)))


def main(deg):
    c, e = remez(deg)
    c32 = c.astype(np.float32)
    print(f"// degree {deg}: minimax relative error {e:.3e} (real coefficients), "
          f"{fp32_eval_error(c32):.3e} (fp32 coefficients, fp32 fma evaluation)")
    for i, ci in enumerate(c32):
        print(f"constexpr float EXP2_C{i} = {float(ci)!r}f;")


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 3)
