"""Minimax polynomial for 2^f on [0, 1), the core of the FMA-pipe exp2.

The kernels compute part of their exponentials 2^x without the special
function unit: Cody and Waite's range reduction splits x = j + f with
j = floor(x) (exact) and f in [0, 1), a polynomial p(f) ~ 2^f gives the
mantissa, and j goes straight into the exponent field.  This module finds
the polynomial of a given degree that minimises the largest RELATIVE error
max |p(f) / 2^f - 1| on [0, 1] by the Remez exchange algorithm (equioscillation
on degree + 2 reference points), in float64.

    python -m kv_cache_sparse_b200.exp2_poly [degree]

prints the coefficients c0 .. c_deg (p(f) = c0 + c1 f + ... , evaluated by
Horner's rule in fp32 on the device) and the error bound.  The constants in
csrc/sm100.cuh were written from its output for degree 3; a CPU test checks
that they agree with a fresh fit and that the bound holds.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(degree: int = 3, iters: int = 30):
    """Coefficients (c0..c_degree) and the equioscillation level E of the
    relative-error minimax approximation of 2^f on [0, 1]."""
    m = degree + 2
    # initial reference: Chebyshev extrema mapped to [0, 1]
    ref = 0.5 - 0.5 * np.cos(np.pi * np.arange(m) / (m - 1))
    grid = np.linspace(0.0, 1.0, 200001)
    coef, E = None, 0.0
    for _ in range(iters):
        # solve p(x_k) - (-1)^k E 2^{x_k} = 2^{x_k} for c and E
        A = np.zeros((m, m))
        for k, x in enumerate(ref):
            A[k, :degree + 1] = x ** np.arange(degree + 1)
            A[k, degree + 1] = -((-1) ** k) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef, E = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        pieces = np.split(np.arange(grid.size), cuts)
        ext = [p[np.argmax(np.abs(err[p]))] for p in pieces]
        if len(ext) < m:
            break
        # keep m alternating extrema, the largest ones
        while len(ext) > m:
            mags = [abs(err[i]) for i in ext]
            drop = 0 if mags[0] < mags[-1] else len(ext) - 1
            ext.pop(drop)
        new_ref = grid[ext]
        if np.allclose(new_ref, ref, atol=1e-12):
            break
        ref = new_ref
    return coef, abs(E)


def max_rel_error(coef, samples: int = 1 << 20) -> float:
    f = np.linspace(0.0, 1.0, samples)
    return float(np.max(np.abs(np.polyval(np.asarray(coef)[::-1], f) / 2.0 ** f - 1.0)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error {e:.3e} (float64 evaluation)")
