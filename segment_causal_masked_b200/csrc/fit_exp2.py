"""Fit the polynomial the attention kernel uses to evaluate 2^f on the FMA pipe.

    python segment_causal_masked_b200/csrc/fit_exp2.py

The kernel computes p = 2^x for x <= 8 in two parts (Cody and Waite's range
reduction): x = j + f with j = round(x) an integer and f in [-1/2, 1/2]; 2^j
is applied by adding j to the exponent field, and 2^f comes from a cubic
P(f) = c0 + c1 f + c2 f^2 + c3 f^3. The coefficients minimise the maximum
relative error max |P(f) / 2^f - 1| over [-1/2, 1/2] (minimax), found here
with the Remez exchange algorithm in float64 and then rounded to float32.

Prints the coefficients (as C hex floats, for the kernel) and the relative
error bound measured on a dense grid after rounding.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 40):
    """Minimax polynomial for 2^f with relative error weight on [LO, HI]."""
    n = degree + 2                                     # reference points
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  solve for (c0..cd, E)
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(a, 2.0 ** x)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of err between sign changes
        sign = np.sign(err)
        breaks = np.flatnonzero(np.diff(sign)) + 1
        pieces = np.split(np.arange(len(grid)), breaks)
        ext = [p[np.argmax(np.abs(err[p]))] for p in pieces if len(p)]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[np.array(ext)]
    return coef


def max_rel_error(coef32: np.ndarray) -> float:
    g = np.linspace(LO, HI, 2_000_001).astype(np.float32)
    p = np.zeros_like(g)
    for c in coef32[::-1]:                              # Horner in float32
        p = (p * g + np.float32(c)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(g.astype(np.float64)) - 1.0)))


def main():
    coef = remez_relative()
    c32 = coef.astype(np.float32)
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c).hex()}f  // {float(c):.9g}")
    print(f"max relative error of the float32 cubic on [-1/2, 1/2]: {max_rel_error(c32):.3e}")


if __name__ == "__main__":
    main()
