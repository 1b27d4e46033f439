"""Fits the polynomial the kernels use for part of their base-2 exponentials.

2^x for x <= 0 is evaluated as 2^r * 2^f with r = round(x) and
f = x - r in [-1/2, 1/2] (Cody and Waite's argument reduction, here with
base 2, where it is exact); 2^f is a polynomial of degree `deg` whose
coefficients minimise the maximum RELATIVE error on [-1/2, 1/2] (Remez
exchange algorithm on the error weighted by 1/2^f).  2^r is applied by adding
r to the float's exponent field.

    python -m kv_cache_sparse_b200.fit_exp2 [deg]

prints the coefficients (lowest order first) and the max relative error of
the polynomial in exact arithmetic.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 40, grid: int = 20001):
    a, b = -0.5, 0.5
    xs = np.linspace(a, b, grid)
    fx = np.exp2(xs)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    ref = np.sort(0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k / (deg + 1)))
    coef = None
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i}  (relative error alternates)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(ref))
        coef = sol[:deg + 1]
        err = (np.polyval(coef[::-1], xs) - fx) / fx
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, grid - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid - 1)
        idx = np.array(sorted(set(idx)))
        # keep deg+2 alternating points with the largest |err|
        pts = [idx[0]]
        for i in idx[1:]:
            if np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > deg + 2:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < deg + 2:
            break
        ref = xs[np.array(pts)]
    err = (np.polyval(coef[::-1], xs) - fx) / fx
    return coef, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e = remez_exp2(deg)
    print("coefficients (c0..c%d):" % deg)
    for v in c:
        print(f"  {np.float32(v)!r:>24}   # {v:.17g}")
    print(f"max relative error {e:.3e}")
