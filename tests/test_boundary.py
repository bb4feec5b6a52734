"""The C-ABI library loads, exports what include/fa.h declares, and rejects bad
arguments before touching a GPU (these run on a machine without one)."""
from __future__ import annotations

import ctypes
import re
import subprocess

import pytest
import torch

from io_aware_tiled_b200 import fa
from io_aware_tiled_b200 import build as fa_build

OK, EINVAL, EALIGN, EDEV, ELAUNCH, EWS, ETIMEOUT = 0, -1, -2, -3, -4, -5, -6


@pytest.fixture(scope="module")
def lib():
    return fa.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = fa.header_functions()
    assert set(names) == {"fa_fwd", "fa_bwd_workspace_bytes", "fa_bwd", "fa_sync_status", "fa_last_error_word",
                          "fa_status_string", "fa_selftest_wait_timeout", "fa_bwd_set_phase_events",
                          "fa_last_cuda_error", "fa_bwd_noalloc", "fa_fwd_kernel_name",
                          "fa_fwd_unfused", "fa_fwd_unfused_workspace_bytes", "fa_bwd_dkdv_kernel_name",
                          "fa_bwd_deterministic", "fa_fwd_bwd_host", "fa_fwd_bwd_host_workspace_bytes",
                          "fa_unit_lists"}
    out = subprocess.run(["nm", "-D", "--defined-only", fa_build.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fa_\w+)", out))
    for n in names:
        assert n in exported, n
        getattr(lib, n)


def test_status_strings(lib):
    for code, name in [(OK, "FA_OK"), (EINVAL, "FA_ERR_INVALID_ARG"), (EALIGN, "FA_ERR_ALIGNMENT"),
                       (EDEV, "FA_ERR_UNSUPPORTED_DEVICE"), (ELAUNCH, "FA_ERR_LAUNCH"),
                       (EWS, "FA_ERR_WORKSPACE"), (ETIMEOUT, "FA_ERR_TIMEOUT"), (-7, "FA_ERR_TOO_LARGE")]:
        assert fa.status_string(code) == name
    assert fa.status_string(42) == "FA_ERR_UNKNOWN"


def test_workspace_bytes(lib):
    # D (fp32 per row, padded to 256 bytes), then the fp32 dQ accumulator
    assert lib.fa_bwd_workspace_bytes(2, 16, 4096, 128) == 2 * 16 * 4096 * 4 + 2 * 16 * 4096 * 128 * 4
    assert lib.fa_bwd_workspace_bytes(8, 12, 1000, 64) == (((8 * 12 * 1000 * 4 + 255) // 256) * 256
                                                           + 8 * 12 * 1000 * 64 * 4)
    assert lib.fa_bwd_workspace_bytes(1, 1, 0, 64) == 0
    assert lib.fa_bwd_workspace_bytes(1, 1, 16, 96) == 0


A = 1 << 20  # fake, 16-byte aligned, never dereferenced: validation stops before any device access


def _fwd(lib, q=A, k=2 * A, v=3 * A, o=4 * A, lse=5 * A, B=1, H=1, N=128, d=64, causal=0, scale=0.0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


def test_forward_rejects_bad_sizes(lib):
    assert _fwd(lib, N=0) == EINVAL
    assert _fwd(lib, N=-3) == EINVAL
    assert _fwd(lib, B=0) == EINVAL
    assert _fwd(lib, H=-1) == EINVAL
    for d in (0, 32, 96, 256):
        assert _fwd(lib, d=d) == EINVAL
    assert _fwd(lib, B=2 ** 16, H=2 ** 16, N=2) == EINVAL  # B*H*N beyond 32-bit rows


def test_forward_rejects_null_misaligned_and_overlap(lib):
    assert _fwd(lib, q=0) == EINVAL
    assert _fwd(lib, lse=0) == EINVAL
    assert _fwd(lib, v=3 * A + 8) == EALIGN
    assert _fwd(lib, o=4 * A + 2) == EALIGN
    assert _fwd(lib, o=A) == EINVAL               # output aliases an input
    assert _fwd(lib, lse=4 * A + 64) == EINVAL    # LSE inside O
    assert _fwd(lib, scale=float("nan")) == EINVAL
    assert _fwd(lib, scale=float("inf")) == EINVAL


def test_forward_without_gpu_reports_unsupported_device(lib):
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) == EDEV


def _bwd(lib, ws=20 * A, ws_bytes=None, B=1, H=1, N=128, d=64, **ptrs):
    p = dict(q=A, k=2 * A, v=3 * A, o=4 * A, do=5 * A, lse=6 * A, dq=7 * A, dk=8 * A, dv=9 * A)
    p.update(ptrs)
    nb = lib.fa_bwd_workspace_bytes(B, H, N, d) if ws_bytes is None else ws_bytes
    return lib.fa_bwd(p["q"], p["k"], p["v"], p["o"], p["do"], p["lse"], p["dq"], p["dk"], p["dv"],
                      B, H, N, d, 1, 0.0, ws, nb, None)


def test_backward_rejects_bad_arguments(lib):
    assert _bwd(lib, N=0) == EINVAL
    assert _bwd(lib, d=80) == EINVAL
    assert _bwd(lib, do=0) == EINVAL
    assert _bwd(lib, dk=8 * A + 4) == EALIGN
    assert _bwd(lib, ws=0) == EWS
    assert _bwd(lib, ws=20 * A + 8) == EWS
    assert _bwd(lib, ws_bytes=16) == EWS
    assert _bwd(lib, dq=A) == EINVAL              # dQ aliases Q
    assert _bwd(lib, dv=8 * A) == EINVAL          # dV aliases dK
    assert _bwd(lib, ws=9 * A) == EWS             # workspace aliases dV


def _unf(lib, ws=20 * A, ws_bytes=None, B=1, H=1, N=128, d=64, causal=0, scale=0.0, **ptrs):
    p = dict(q=A, k=2 * A, v=3 * A, o=4 * A, lse=5 * A)
    p.update(ptrs)
    nb = lib.fa_fwd_unfused_workspace_bytes(B, H, N, d) if ws_bytes is None else ws_bytes
    return lib.fa_fwd_unfused(p["q"], p["k"], p["v"], p["o"], p["lse"], B, H, N, d, causal, scale, ws, nb, None)


def test_unfused_workspace_bytes(lib):
    # S and then P, 16-bit, [B*H][Nr][Nr] with Nr = N rounded up to 128
    assert lib.fa_fwd_unfused_workspace_bytes(2, 16, 4096, 128) == 2 * 16 * 4096 * 4096 * 2
    assert lib.fa_fwd_unfused_workspace_bytes(8, 12, 1000, 64) == 8 * 12 * 1024 * 1024 * 2
    assert lib.fa_fwd_unfused_workspace_bytes(1, 1, 1, 64) == 128 * 128 * 2
    assert lib.fa_fwd_unfused_workspace_bytes(1, 1, 0, 64) == 0
    assert lib.fa_fwd_unfused_workspace_bytes(1, 1, 16, 96) == 0


def test_unfused_rejects_bad_arguments(lib):
    assert _unf(lib, N=0) == EINVAL
    assert _unf(lib, d=32) == EINVAL
    assert _unf(lib, q=0) == EINVAL
    assert _unf(lib, o=4 * A + 2) == EALIGN
    assert _unf(lib, scale=float("nan")) == EINVAL
    assert _unf(lib, o=2 * A) == EINVAL            # O aliases K
    assert _unf(lib, ws=0) == EWS
    assert _unf(lib, ws=20 * A + 8) == EWS
    assert _unf(lib, ws_bytes=1024) == EWS
    assert _unf(lib, ws=3 * A) == EWS              # workspace aliases V
    if not torch.cuda.is_available():
        assert _unf(lib) == EDEV


def test_dkdv_kernel_name():
    # pure host logic: no device needed
    assert fa.dkdv_kernel_name(128) == "fa_bwd_fused_kernel"
    assert fa.dkdv_kernel_name(64) == "fa_bwd_fused_kernel"
    assert fa.dkdv_kernel_name(128, deterministic=True) == "fa_bwd_dkdv_kernel"
    assert fa.backward_kernel_names(64) == ("fa_bwd_preprocess_kernel", "fa_bwd_fused_kernel",
                                            "fa_bwd_dq_convert_kernel")
    assert fa.backward_kernel_names(128, True) == ("fa_bwd_preprocess_kernel", "fa_bwd_dkdv_kernel",
                                                   "fa_bwd_dq_kernel")
    with pytest.raises(RuntimeError):
        fa.dkdv_kernel_name(96)


def _bwd_det(lib, ws=20 * A, ws_bytes=None, B=1, H=1, N=128, d=64, **ptrs):
    p = dict(q=A, k=2 * A, v=3 * A, o=4 * A, do=5 * A, lse=6 * A, dq=7 * A, dk=8 * A, dv=9 * A)
    p.update(ptrs)
    nb = ((B * H * N * 4 + 255) // 256) * 256 if ws_bytes is None else ws_bytes
    return lib.fa_bwd_deterministic(p["q"], p["k"], p["v"], p["o"], p["do"], p["lse"], p["dq"], p["dk"], p["dv"],
                                    B, H, N, d, 1, 0.0, ws, nb, None)


def test_deterministic_backward_needs_only_the_d_part(lib):
    """fa_bwd_deterministic takes the same arguments as fa_bwd but uses only
    the D part of the workspace; fa_bwd needs D and the dQ accumulator."""
    d_bytes = ((128 * 4 + 255) // 256) * 256
    assert _bwd_det(lib, ws_bytes=d_bytes - 16) == EWS
    assert _bwd(lib, ws_bytes=d_bytes) == EWS
    assert _bwd_det(lib, N=0) == EINVAL
    assert _bwd_det(lib, dk=8 * A + 4) == EALIGN
    assert _bwd_det(lib, dq=A) == EINVAL
    if not torch.cuda.is_available():
        assert _bwd_det(lib, ws_bytes=d_bytes) == EDEV   # valid arguments: stops at the device check
        assert _bwd(lib) == EDEV


def test_selftest_rejects_bad_limit(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == EINVAL
    assert lib.fa_selftest_wait_timeout(10_000_001, None) == EINVAL


def test_python_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)
    with pytest.raises(ValueError):
        fa.forward(q.float(), q.float(), q.float())


def test_host_pipeline_workspace_bytes(lib):
    """Three slots, each one head group's Q, K, V, dO, O, dQ, dK, dV (bf16), LSE
    (fp32) and backward workspace, every region rounded up to 256 bytes."""
    def up(x):
        return (x + 255) // 256 * 256

    def slot(hc, N, d):
        t, l = up(hc * N * d * 2), up(hc * N * 4)
        return 8 * t + l + up(lib.fa_bwd_workspace_bytes(1, hc, N, d))

    assert lib.fa_fwd_bwd_host_workspace_bytes(2, 16, 4096, 128, 8) == 3 * slot(4, 4096, 128)
    assert lib.fa_fwd_bwd_host_workspace_bytes(2, 3, 300, 64, 4) == 3 * slot(2, 300, 64)  # 6 heads -> groups of 2
    assert lib.fa_fwd_bwd_host_workspace_bytes(1, 2, 100, 64, 50) == 3 * slot(1, 100, 64)  # clamped to B*H
    assert lib.fa_fwd_bwd_host_workspace_bytes(1, 1, 100, 64, 0) == 0
    assert lib.fa_fwd_bwd_host_workspace_bytes(1, 1, 0, 64, 1) == 0


def _host(lib, ws=30 * A, ws_bytes=None, B=1, H=2, N=128, d=64, groups=2, **ptrs):
    p = dict(q=A, k=2 * A, v=3 * A, do=4 * A, o=5 * A, lse=6 * A, dq=7 * A, dk=8 * A, dv=9 * A)
    p.update(ptrs)
    nb = lib.fa_fwd_bwd_host_workspace_bytes(B, H, N, d, groups) if ws_bytes is None else ws_bytes
    return lib.fa_fwd_bwd_host(p["q"], p["k"], p["v"], p["do"], p["o"], p["lse"], p["dq"], p["dk"], p["dv"],
                               B, H, N, d, 0, 0.0, groups, ws, nb, None)


def test_host_pipeline_rejects_bad_arguments(lib):
    assert _host(lib, N=0) == EINVAL
    assert _host(lib, d=32) == EINVAL
    assert _host(lib, groups=0) == EINVAL
    assert _host(lib, q=0) == EINVAL
    assert _host(lib, lse=0) == EINVAL
    assert _host(lib, ws=0) == EWS
    assert _host(lib, ws=30 * A + 8) == EWS
    assert _host(lib, ws_bytes=1024) == EWS
    assert _host(lib, o=A) == EINVAL              # O aliases Q
    assert _host(lib, dv=8 * A) == EINVAL         # dV aliases dK
    if not torch.cuda.is_available():
        assert _host(lib) == EDEV                 # valid arguments: stops at the device check
