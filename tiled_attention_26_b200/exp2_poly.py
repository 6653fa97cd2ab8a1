"""Coefficients of the polynomial that evaluates 2^f on the FMA pipe for part of the softmax.

Method (Cody-Waite style range reduction followed by a minimax polynomial, derived here):
  x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2]; 2^x = 2^n * 2^f, where 2^n is
  applied by adding n to the exponent field and 2^f is a polynomial p(f).
  p minimises the maximum RELATIVE error |p(f) / 2^f - 1| over [-1/2, 1/2] (Remez exchange on
  the relative error, starting from Chebyshev nodes), with p(0) free.

Running this file prints the coefficients (highest degree first) and the achieved error; the
values are copied into prefill.cuh and checked by tests/test_exp2_poly.py.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int, iters: int = 30):
    lo, hi = -0.5, 0.5
    n = degree + 2
    # Chebyshev extrema as the starting reference
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i * E * 2^x_i   (relative equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :degree + 1] = xi ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0 and abs(err[j]) > 1e-30:
                idx.append(j)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        cand = grid[idx]
        vals = err[idx]
        # keep alternating extrema with the largest magnitude
        keep = [0]
        for j in range(1, len(cand)):
            if np.sign(vals[j]) == np.sign(vals[keep[-1]]):
                if abs(vals[j]) > abs(vals[keep[-1]]):
                    keep[-1] = j
            else:
                keep.append(j)
        if len(keep) >= n:
            while len(keep) > n:
                if abs(vals[keep[0]]) < abs(vals[keep[-1]]):
                    keep.pop(0)
                else:
                    keep.pop()
            x = cand[keep]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    for deg in (3, 4):
        c, e = remez_exp2(deg)
        print(f"degree {deg}: max rel err {e:.3e}")
        print("  coefficients c0..c%d:" % deg, ", ".join(f"{v:.9e}" for v in c))
        print("  float32:", ", ".join(repr(float(np.float32(v))) for v in c))
