"""exp2_poly3 (the forward softmax's FMA-pipe exponential, fa_device.cuh):
its constants are the Remez fit that csrc/fit_exp2_poly.py computes, and the
float32 evaluation it performs stays within 7.5e-5 relative of 2^t for t in
[-125, 8] (the softmax's arguments stay <= 8), with no NaN or negative value for masked
(-inf) scores.  CPU only: numpy reproduces the kernel's float32 steps."""
from __future__ import annotations

import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "io_aware_tiled_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_constants():
    src = open(os.path.join(CSRC, "fa_device.cuh"), encoding="utf-8").read()
    body = src[src.index("float exp2_poly3(float t)"):]
    body = body[:body.index("}")]
    clamp = float(re.search(r"fmaxf\(t, (-?[0-9.]+)f\)", body).group(1))
    poly = re.search(r"fmaf\(fmaf\(fmaf\(([0-9.e-]+)f, f, ([0-9.e-]+)f\), f, ([0-9.e-]+)f\), f, ([0-9.e-]+)f\)", body)
    c3, c2, c1, c0 = (np.float32(float(g)) for g in poly.groups())
    return clamp, np.array([c0, c1, c2, c3], dtype=np.float32)


def test_constants_are_the_remez_fit():
    fit = _fit_module()
    _, c_kernel = _kernel_constants()
    c_fit = fit.remez_exp2().astype(np.float32)
    assert np.array_equal(c_kernel, c_fit), (c_kernel, c_fit)


def test_relative_error_bound_on_softmax_arguments():
    fit = _fit_module()
    clamp, c = _kernel_constants()
    assert clamp == -126.0
    t = np.concatenate([np.linspace(-125.0, 8.0, 3_000_001), np.arange(-125, 8, dtype=np.float64) + 0.5,
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    y = fit.emulate_f32(t, c).astype(np.float64)
    rel = np.abs(y / np.exp2(t.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5, rel.max()
    # below -125 the result may be subnormal (no implicit bit, not accurate):
    # only that it is finite, non-negative and below 2^-124 matters
    tt = np.linspace(-126.5, -125.0, 100001).astype(np.float32)
    yy = fit.emulate_f32(tt, c).astype(np.float64)
    assert np.isfinite(yy).all() and (yy >= 0).all() and (yy <= 2.0 ** -124).all()
    # 2^0 and the powers of two come out within the same bound
    assert abs(float(fit.emulate_f32(np.array([0.0], np.float32), c)[0]) - 1.0) <= 7.5e-5


def test_masked_scores_give_tiny_nonnegative_values():
    fit = _fit_module()
    _, c = _kernel_constants()
    t = np.array([-np.inf, -1e30, -1000.0, -127.0, -126.6, -126.5, -126.0], dtype=np.float32)
    y = fit.emulate_f32(t, c)
    assert np.isfinite(y).all() and (y >= 0).all() and (y <= 2.0 ** -125).all()
    # the same steps with the clamp at -127 would wrap the exponent field into NaN
    t127 = np.array([-127.0], dtype=np.float32)
    r = (t127 + np.float32(12582912.0)).astype(np.float32)
    p = np.float32(c[0])  # f = 0
    wrapped = (np.array([p]).view(np.int32) + (r.view(np.int32) << 23)).view(np.float32)
    assert np.isnan(wrapped).all()


def test_paired_form_uses_the_same_steps():
    """exp2_poly3_x2 (two values on the paired fp32 instructions) repeats the
    scalar form's clamp, rounding constant and polynomial lane by lane."""
    src = open(os.path.join(CSRC, "fa_device.cuh"), encoding="utf-8").read()
    body = src[src.index("void exp2_poly3_x2("):]
    body = body[:body.index("\n}\n")]
    clamp, c = _kernel_constants()
    assert body.count(f"fmaxf(t0, {clamp:.0f}.f)") == 1 and body.count(f"fmaxf(t1, {clamp:.0f}.f)") == 1
    pairs = re.findall(r"f2_make\(([0-9.e-]+)f, ([0-9.e-]+)f\)", body)
    vals = {float(a) for a, b in pairs if a == b}
    assert all(a == b for a, b in pairs)
    assert 12582912.0 in vals
    for k in range(4):
        assert any(np.float32(v) == c[k] for v in vals), c[k]
    assert "f2_fma(f2_fma(f2_fma(c3, f, c2), f, c1), f, c0)" in body
    scalar = src[src.index("float exp2_poly3(float t)"):]
    assert "12582912.f" in scalar[:scalar.index("}")]
