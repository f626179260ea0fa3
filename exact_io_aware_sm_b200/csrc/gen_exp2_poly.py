"""Coefficients of the polynomial exp2 used by the prefill softmax.

2^x is split as 2^j * 2^f with j = rint(x) and f = x - j in [-1/2, 1/2]
(Cody and Waite's argument reduction, "Software Manual for the Elementary
Functions", 1980).  2^f is approximated by a degree-3 polynomial whose
coefficients minimise the maximum relative error on [-1/2, 1/2], found with
the Remez exchange algorithm (E. Remez, 1934) on the relative-error
weighting.  The kernel evaluates it with fused multiply-adds in Horner form
and adds j to the exponent field.

    python -m exact_io_aware_sm_b200.csrc.gen_exp2_poly

prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the error bound.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 40):
    n = degree + 2
    # initial reference: Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n)
    x = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E * 2^x_i  (relative error alternation)
        f = np.exp2(x)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * f[i]
        sol = np.linalg.solve(A, f)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: the extrema of the error between sign changes
        idx = [0]
        s = np.sign(err)
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep n alternating points with the largest errors
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}  ({ci:.17g})")
    print(f"max relative error on [{LO}, {HI}] (exact arithmetic): {e:.3e}")
