"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp32 accumulation):
  O    : max over elements of |O_gpu - O_oracle| - ulp_bf16(O_oracle)/2 <= 1e-2, and
         ||O_gpu - bf16(O_oracle)||_F / ||bf16(O_oracle)||_F <= 5e-3
  LSE  : max |LSE_gpu - LSE_oracle| <= 1e-3
  dQ, dK, dV : ||g_gpu - g_oracle||_F / ||g_oracle||_F <= 1e-2
O is a bf16 output, so no implementation can be nearer to the exact value
than half a bf16 spacing (1/128 for |O| in [2, 4)); the 1e-2 max-abs budget
applies to the arithmetic error beyond that format floor.  A one-spacing
rounding flip next to a rounding midpoint therefore passes, an arithmetic
error of 1e-2 does not.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_FROB = 5e-3
LSE_ABS = 1e-3
GRAD_REL_FROB = 1e-2


def to_bf16_np(x: np.ndarray) -> np.ndarray:
    """Round an fp64 array to bf16 (nearest even) and return it as fp64."""
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_frob(x, ref) -> float:
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x, ref) -> float:
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def half_ulp_bf16(x) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    x = np.abs(np.asarray(x, np.float64))
    _, e = np.frexp(x)  # x = m * 2**e, m in [0.5, 1)
    return np.where(x > 0, np.ldexp(1.0, e - 9), 0.0)


def o_excess_error(o_gpu, o_oracle) -> float:
    """max |O_gpu - O_oracle| beyond the bf16 output's half spacing."""
    o_gpu, o_oracle = np.asarray(o_gpu, np.float64), np.asarray(o_oracle, np.float64)
    if not o_gpu.size:
        return 0.0
    return float(np.max(np.abs(o_gpu - o_oracle) - half_ulp_bf16(o_oracle)))


# Every O, LSE and gradient comparison made in this session, for the summary
# pytest prints at the end (tests/conftest.py): what was compared and the
# measured errors, so the share of each bound in use is visible.
RECORD: list = []


def check_o(o_gpu, o_oracle, what=""):
    ma = o_excess_error(o_gpu, o_oracle)
    o_bf16 = to_bf16_np(o_oracle)
    plain = max_abs(o_gpu, o_bf16)  # against the oracle rounded to bf16, no allowance
    rf = rel_frob(o_gpu, o_bf16)
    RECORD.append(("O", what, {"max_abs_vs_bf16_oracle": plain, "max_abs_beyond_half_ulp": ma, "rel_frob": rf}))
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite O"
    assert ma <= O_MAX_ABS, f"{what}: O max-abs beyond the bf16 half spacing {ma:.3e} > {O_MAX_ABS}"
    assert rf <= O_REL_FROB, f"{what}: O rel-frob {rf:.3e} > {O_REL_FROB}"
    return ma, rf


def check_lse(lse_gpu, lse_oracle, what=""):
    ma = max_abs(lse_gpu, lse_oracle)
    RECORD.append(("LSE", what, {"max_abs": ma}))
    assert np.isfinite(lse_gpu).all(), f"{what}: non-finite LSE"
    assert ma <= LSE_ABS, f"{what}: LSE max-abs {ma:.3e} > {LSE_ABS}"
    return ma


def check_grad(g_gpu, g_oracle, name, what=""):
    rf = rel_frob(g_gpu, g_oracle)
    RECORD.append((name, what, {"rel_frob": rf}))
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite {name}"
    assert rf <= GRAD_REL_FROB, f"{what}: {name} rel-frob {rf:.3e} > {GRAD_REL_FROB}"
    return rf


def assert_same_up_to_summation_order(a: torch.Tensor, b: torch.Tensor, what=""):
    """Two bf16 results of the same products whose fp32 partial sums were
    added in different orders (the default backward's dQ): each element may
    differ by one bf16 rounding step (2^-7 relative) plus an absolute floor of
    1e-6 x max|b| for elements near zero, where fp32 cancellation among the
    partial sums leaves a larger relative difference; over the tensor, the
    relative Frobenius difference stays below 1e-3."""
    x, y = a.detach().double().cpu(), b.detach().double().cpu()
    assert x.shape == y.shape, what
    assert torch.isfinite(x).all(), f"{what}: non-finite"
    scale = float(y.abs().max()) if y.numel() else 0.0
    bound = torch.maximum(x.abs(), y.abs()) * 2.0 ** -7 + 1e-6 * scale
    worst = float((x - y).abs().sub(bound).max()) if x.numel() else 0.0
    assert worst <= 0.0, f"{what}: differs beyond one bf16 step by {worst:.3e}"
    rf = float((x - y).norm() / (y.norm() if float(y.norm()) > 0 else 1.0))
    assert rf <= 1e-3, f"{what}: rel-frob difference {rf:.3e}"
    return rf
