"""Fit the polynomial behind the kernels' FMA-pipe exp2 (exp2_fma2 in
sm100_ptx.cuh) and print its coefficients.

Method: Cody-Waite style range reduction x = n + f with n = round-to-nearest(x),
f in [-1/2, 1/2], so 2^x = 2^n * 2^f; 2^n is applied by adding n to the fp32
exponent field.  2^f is a degree-`deg` polynomial with its constant term fixed
at 1 (so 2^n comes out exact for integer x and the clamp at x = -127 gives an
exact 0), fitted by the Remez exchange algorithm to minimise the maximum
*relative* error max |p(f) - 2^f| / 2^f on [-1/2, 1/2].

Run:  python exact_attention_109_b200/csrc/exp2_poly_fit.py [deg]
"""
from __future__ import annotations

import sys

import numpy as np


def fit(deg: int = 3, iters: int = 60):
    """Coefficients a_1..a_deg of p(f) = 1 + sum a_k f^k, and the max rel error."""
    lo, hi = -0.5, 0.5
    m = deg + 1                      # unknowns: a_1..a_deg and the level E
    # initial reference: Chebyshev-like points, avoiding the fixed zero at 0
    ref = np.cos(np.pi * (np.arange(m) + 0.5) / m)[::-1] * 0.5
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        A = np.zeros((m, m))
        rhs = np.exp2(ref) - 1.0
        for i, x in enumerate(ref):
            A[i, :deg] = [x ** k for k in range(1, deg + 1)]
            A[i, deg] = -((-1.0) ** i) * np.exp2(x)
        sol = np.linalg.solve(A, rhs)
        coef = sol[:deg]
        err = (1.0 + sum(c * grid ** (k + 1) for k, c in enumerate(coef))
               - np.exp2(grid)) / np.exp2(grid)
        # new reference: the extremum of each sign-run of the error
        sign = np.sign(err)
        idx = []
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sign[k] != sign[start]:
                seg = slice(start, k)
                j = start + int(np.argmax(np.abs(err[seg])))
                if abs(err[j]) > 0:
                    idx.append(j)
                start = k
        # keep the m largest alternating extrema
        while len(idx) > m:
            drop = min(range(len(idx)), key=lambda t: abs(err[idx[t]]))
            idx.pop(drop)
        if len(idx) < m:
            break
        new = grid[idx]
        if np.allclose(new, ref, atol=1e-12):
            break
        ref = new
    err = (1.0 + sum(c * grid ** (k + 1) for k, c in enumerate(coef))
           - np.exp2(grid)) / np.exp2(grid)
    return [float(c) for c in coef], float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, e = fit(deg)
    print(f"degree {deg}: max relative error {e:.3e}")
    for k, c in enumerate(coef, start=1):
        print(f"a{k} = {np.float32(c)!r}  ({c:.17g})")
