"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (``io_aware_tiled_b200`` and
its CUDA library) never imports it, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module only marshals numpy arrays.  Every function takes the exact bf16 input
values widened to float64 and returns float64.

What is computed, and the pages it follows, is stated in ``oracle.c``'s
header.  Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (worked example, closed forms, invariants,
brute force, finite differences, a library special case).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` with gcc (OpenMP, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i, d = ctypes.c_int, ctypes.c_double
        lib.oracle_forward.argtypes = [_dp, _dp, _dp, i, i, i, i, i, d, _dp, _dp]
        lib.oracle_probs.argtypes = [_dp, _dp, i, i, i, i, i, d, i, _dp]
        lib.oracle_forward_rows.argtypes = [_dp, _dp, _dp, i, i, i, i, i, d, i, _i64p, _dp, _dp]
        lib.oracle_backward.argtypes = [_dp, _dp, _dp, _dp, _dp, i, i, i, i, i, d,
                                        _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_backward_sampled.argtypes = [_dp, _dp, _dp, _dp, _dp, i, i, i, i, i, d,
                                                i, i, _i64p, i, _i64p, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [i]
        for f in (lib.oracle_forward, lib.oracle_probs, lib.oracle_forward_rows,
                  lib.oracle_backward, lib.oracle_backward_sampled):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(_dp)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc}")


def _shape4(q) -> tuple[int, int, int, int]:
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    return tuple(int(s) for s in q.shape)  # type: ignore[return-value]


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def forward(q, k, v, causal: bool, scale: float):
    """O [B,H,N,d] and LSE [B,H,N] from the materialised definition."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape4(q)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    _check(_load().oracle_forward(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, int(bool(causal)),
                                  float(scale), _ptr(o), _ptr(lse)), "forward")
    return o, lse


def probs(q, k, causal: bool, scale: float, bh: int = 0):
    """The N x N attention probabilities P of head ``bh`` (flattened b*H+h)."""
    q, k = _f64(q), _f64(k)
    B, H, N, d = _shape4(q)
    p = np.empty((N, N), dtype=np.float64)
    _check(_load().oracle_probs(_ptr(q), _ptr(k), B, H, N, d, int(bool(causal)), float(scale),
                                int(bh), _ptr(p)), "probs")
    return p


def forward_rows(q, k, v, causal: bool, scale: float, rows):
    """O and LSE of the listed rows only; ``rows`` holds flat indices bh*N + i."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape4(q)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty((rows.size,), dtype=np.float64)
    _check(_load().oracle_forward_rows(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, int(bool(causal)),
                                       float(scale), int(rows.size), rows.ctypes.data_as(_i64p),
                                       _ptr(o), _ptr(lse)), "forward_rows")
    return o, lse


def backward(q, k, v, do, causal: bool, scale: float, o_for_d=None):
    """Full backward.  Returns a dict with dq, dk, dv, D (definitional, or the
    rowsum form over ``o_for_d`` when given), D_rowsum (over the oracle's own
    O), o and lse."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = _shape4(q)
    ofd = None if o_for_d is None else _f64(o_for_d)
    out = {n: np.empty_like(q) for n in ("dq", "dk", "dv", "o")}
    for n in ("D", "D_rowsum", "lse"):
        out[n] = np.empty((B, H, N), dtype=np.float64)
    _check(_load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(ofd), B, H, N, d,
                                   int(bool(causal)), float(scale), _ptr(out["dq"]),
                                   _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["D"]),
                                   _ptr(out["D_rowsum"]), _ptr(out["o"]), _ptr(out["lse"])),
           "backward")
    return out


def backward_sampled(q, k, v, do, causal: bool, scale: float, bh: int, q_rows, k_rows,
                     o_for_d=None):
    """Backward of head ``bh`` restricted to sampled rows: dq for ``q_rows``,
    dk and dv for ``k_rows``, plus that head's lse and D for every row."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = _shape4(q)
    ofd = None if o_for_d is None else _f64(o_for_d)
    qr = np.ascontiguousarray(np.asarray(q_rows, dtype=np.int64))
    kr = np.ascontiguousarray(np.asarray(k_rows, dtype=np.int64))
    out = {
        "dq": np.empty((qr.size, d)), "dk": np.empty((kr.size, d)), "dv": np.empty((kr.size, d)),
        "lse": np.empty((N,)), "D": np.empty((N,)),
    }
    _check(_load().oracle_backward_sampled(
        _ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(ofd), B, H, N, d, int(bool(causal)),
        float(scale), int(bh), int(qr.size), qr.ctypes.data_as(_i64p), int(kr.size),
        kr.ctypes.data_as(_i64p), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
        _ptr(out["lse"]), _ptr(out["D"])), "backward_sampled")
    return out
