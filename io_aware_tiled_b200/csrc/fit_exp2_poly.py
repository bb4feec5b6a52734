"""Fits the polynomial of exp2_poly3 (fa_device.cuh): the degree-3 polynomial
p(f) ~ 2^f on [-1/2, 1/2] with the least maximum RELATIVE error, by the Remez
exchange algorithm (E. Remez, 1934): solve for coefficients that make the
relative error equioscillate on n + 2 reference points, move the references
to the extrema of the new error, repeat.  Range reduction is Cody and Waite's
(W. Cody, W. Waite, Software Manual for the Elementary Functions, 1980):
2^t = 2^j * 2^f with j = rint(t), f = t - j.

Run it to print the coefficients as float32 and the error of the float32
evaluation that exp2_poly3 performs; tests/test_exp2_poly.py checks that the
kernel's constants are this fit's.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def remez_exp2(deg: int = DEGREE, a: float = -0.5, b: float = 0.5, iters: int = 30, grid: int = 200001):
    n = deg + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))  # Chebyshev extrema
    g = np.linspace(a, b, grid)
    c = None
    for _ in range(iters):
        m = np.zeros((n, n))
        for i in range(n):
            m[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            m[i, deg + 1] = (-1) ** i * 2.0 ** x[i]  # p(x_i) + (-1)^i E 2^x_i = 2^x_i
        c = np.linalg.solve(m, 2.0 ** x)[:deg + 1]
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        sign_change = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], sign_change + 1, [grid]])
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = g[ext]
    return c


def emulate_f32(t: np.ndarray, c32: np.ndarray) -> np.ndarray:
    """exp2_poly3's float32 steps (separate multiply and add instead of fma)."""
    t = np.maximum(t.astype(np.float32), np.float32(-126.0))
    r = (t + np.float32(12582912.0)).astype(np.float32)  # 1.5 * 2^23: rint(t) in the low mantissa bits
    f = (t - (r - np.float32(12582912.0))).astype(np.float32)
    p = np.float32(c32[-1]) * np.ones_like(f)
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + np.float32(c32[k])).astype(np.float32)
    return (p.view(np.int32) + (r.view(np.int32) << 23)).view(np.float32)


if __name__ == "__main__":
    c32 = remez_exp2().astype(np.float32)
    t = np.linspace(-30.0, 8.0, 2000001).astype(np.float32)
    rel = float(np.abs(emulate_f32(t, c32).astype(np.float64) / np.exp2(t.astype(np.float64)) - 1.0).max())
    print("coefficients c0..c3 (float32):", ", ".join(f"{float(v):.10g}f" for v in c32))
    print(f"max relative error of the float32 evaluation on [-30, 8]: {rel:.3e}")
