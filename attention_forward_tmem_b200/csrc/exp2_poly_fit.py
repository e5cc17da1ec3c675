"""Fit the polynomial behind the FMA-pipe exp2 of the softmax.

2^x is evaluated as 2^n * P(f) with n = round(x), f = x - n in [-1/2, 1/2]
(Cody & Waite range reduction, "Software Manual for the Elementary
Functions", 1980).  P is the degree-3 polynomial minimising the maximum
RELATIVE error of P(f) against 2^f on [-1/2, 1/2], found with the Remez
exchange algorithm (equioscillation of the weighted error on n + 2 points).

Run:  python exp2_poly_fit.py   -> prints the coefficients and the error bound;
the kernel's constants (sm100_ptx.cuh, exp2_poly) must match this output.
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    f = lambda t: np.exp2(t)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_j c_j t^j + (-1)^i E f(t_i) = f(t_i)   (relative weighting)
        A = np.zeros((deg + 2, deg + 2))
        for i, t in enumerate(ref):
            A[i, :deg + 1] = t ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(t)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        # keep deg + 2 alternating extrema with the largest magnitude
        pts = list(idx)
        while len(pts) > deg + 2:
            e = np.abs(err[pts])
            # drop the smallest among adjacent same-sign pairs, else the smallest end
            dropped = False
            for j in range(len(pts) - 1):
                if np.sign(err[pts[j]]) == np.sign(err[pts[j + 1]]):
                    pts.pop(j if e[j] < e[j + 1] else j + 1)
                    dropped = True
                    break
            if not dropped:
                pts.pop(0 if e[0] < e[-1] else len(pts) - 1)
        ref = grid[pts]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3 (P(f) = c0 + c1 f + c2 f^2 + c3 f^3):")
    for v in c:
        print(f"  {np.float32(v)!r}  ({v:.10e})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
