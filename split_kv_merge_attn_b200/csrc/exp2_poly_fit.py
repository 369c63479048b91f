"""Coefficients of the FMA-pipe exp2 used by the prefill softmax (prefill.cuh).

2^x is evaluated as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction; the scaling by 2^n is an addition to the
exponent field).  2^f is a polynomial of degree 3 whose coefficients minimise
the maximum RELATIVE error over [-1/2, 1/2]: the Remez exchange algorithm
(equioscillation of the weighted error at degree + 2 points), written out
here with numpy.  Run it to print the coefficients and the error bound that
prefill.cuh states:

    python split_kv_merge_attn_b200/csrc/exp2_poly_fit.py
"""
from __future__ import annotations

import numpy as np


def remez_relative(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    f = lambda x: np.exp2(x)
    # Chebyshev extrema as the first reference
    k = np.arange(deg + 2)
    ref = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    E = 0.0
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i): solve for the coefficients and E
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        coef, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(coef[::-1], grid) - f(grid)) / f(grid)
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]))
        ext = [a + int(np.argmax(np.abs(err[a:b]))) for a, b in zip(idx[:-1], idx[1:])]
        if len(ext) < deg + 2:
            break
        # keep deg + 2 alternating extrema with the largest errors
        while len(ext) > deg + 2:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else -1
            ext.pop(drop)
        ref = grid[ext]
    err = (np.polyval(coef[::-1], grid) - f(grid)) / f(grid)
    return coef, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_relative()
    for i, ci in enumerate(c):
        print(f"c{i} = {float(np.float32(ci))!r}")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
