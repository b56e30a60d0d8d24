"""Fit the polynomial the kernels use for 2^f on f in [-1/2, 1/2].

The forward kernel evaluates part of its exponentials without the special
function unit: 2^x = 2^n * 2^f with n = round(x) and f = x - n, and 2^f from a
degree-3 polynomial whose coefficients this script computes with a Remez
exchange that minimises the maximum RELATIVE error (float64), then rounds to
float32.  Run:  python -m exact_io_aware_100_b200.fit_exp2_poly
"""
from __future__ import annotations

import numpy as np


def remez_relative(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.where(np.diff(sign) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [grid.size]])
        ext = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            j = a + np.argmax(np.abs(err[a:b]))
            ext.append(j)
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext.pop(0)
            else:
                ext.pop()
        x = grid[np.array(ext)]
    c32 = c.astype(np.float32)
    err32 = (np.polyval(c32.astype(np.float64)[::-1], grid) - f(grid)) / f(grid)
    return c32, float(np.abs(err32).max())


if __name__ == "__main__":
    c, e = remez_relative()
    for i, v in enumerate(c):
        print(f"C{i} = {float(v)!r}  ({float(v).hex()})")
    print(f"max relative error (float32 coefficients, exact arithmetic): {e:.3e}")
