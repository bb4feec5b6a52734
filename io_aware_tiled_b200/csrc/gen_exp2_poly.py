"""Fits the polynomial the kernels use for 2^f on f in [-1/2, 1/2].

Method: Cody-Waite style range reduction (x = n + f, n = round(x), so
2^x = 2^n * 2^f with 2^n assembled in the exponent bits) and a polynomial for
2^f whose coefficients minimise the maximum RELATIVE error on [-1/2, 1/2]
(Remez exchange, written here, started on Chebyshev extrema).  Prints the
coefficients as float32 literals and the achieved error.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, iters: int = 60):
    """Unknowns c0..c_deg and the levelled error E, on degree + 2 points."""
    a, b = -0.5, 0.5
    k = degree + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(k)[::-1] / (k - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # sum_j c_j x_i^j - 2^x_i = (-1)^i E 2^x_i
        A = np.zeros((k, k))
        rhs = np.zeros(k)
        for i, xi in enumerate(x):
            t = 2.0 ** xi
            for j in range(degree + 1):
                A[i, j] = xi ** j
            A[i, degree + 1] = -((-1) ** i) * t
            rhs[i] = t
        sol = np.linalg.solve(A, rhs)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: one extremum of |err| per run of constant sign
        pts = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or np.sign(err[i]) != np.sign(err[start]):
                j = start + int(np.argmax(np.abs(err[start:i])))
                pts.append(j)
                start = i
        while len(pts) > k:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) == k:
            x = grid[pts]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(grid)
    for ci in c32[::-1]:
        p = p * grid + ci  # Horner in float32, as the kernel does
    rel = np.max(np.abs(p.astype(np.float64) - 2.0 ** grid.astype(np.float64)) / 2.0 ** grid.astype(np.float64))
    print("max relative error (fp64 coefficients):", e)
    print("max relative error (fp32 Horner):", rel)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}  ({np.float32(ci).view(np.uint32):#010x})")
