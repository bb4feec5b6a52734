"""Thin Python binding of libfa.so (argument marshalling only).

Every step of the attention path runs in the library's sm_100a kernels;
torch supplies device memory and the current CUDA stream.  There is no CPU
fallback: if the library is missing or the device is not an sm_100 GPU, the
calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

from . import build as _build

_HEADER = os.path.join(_build.INCLUDE, "fa.h")

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_ALIGNMENT = -2
FA_ERR_UNSUPPORTED_DEVICE = -3
FA_ERR_LAUNCH = -4
FA_ERR_WORKSPACE = -5
FA_ERR_TIMEOUT = -6
FA_ERR_TOO_LARGE = -7
NOALLOC_MAX_ROWS = 1 << 20


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        extra = ""
        if status == FA_ERR_LAUNCH:
            extra = f", cudaError {load_library().fa_last_cuda_error()}"
        super().__init__(f"{what}: {status_string(status)} ({status}{extra})")


_lib = None


def library_path() -> str:
    return _build.LIB


def load_library(build_if_missing: bool = True):
    """Load libfa.so (building it first if it is missing or older than its sources)."""
    global _lib
    if _lib is None:
        if build_if_missing and _build.stale():
            _build.build()
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"libfa.so is not built ({_build.LIB}); run io_aware_tiled_b200.build.build()")
        lib = ctypes.CDLL(_build.LIB)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
        lib.fa_fwd.restype = i
        lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
        lib.fa_bwd_workspace_bytes.restype = sz
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
        lib.fa_bwd.restype = i
        lib.fa_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
        lib.fa_bwd_deterministic.restype = i
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
        lib.fa_bwd_noalloc.restype = i
        lib.fa_sync_status.argtypes = [vp]
        lib.fa_sync_status.restype = i
        lib.fa_last_error_word.argtypes = []
        lib.fa_last_error_word.restype = ctypes.c_uint
        lib.fa_last_cuda_error.argtypes = []
        lib.fa_last_cuda_error.restype = i
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_fwd_unfused_workspace_bytes.argtypes = [i, i, i, i]
        lib.fa_fwd_unfused_workspace_bytes.restype = sz
        lib.fa_fwd_unfused.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
        lib.fa_fwd_unfused.restype = i
        lib.fa_bwd_dkdv_kernel_name.argtypes = [i]
        lib.fa_bwd_dkdv_kernel_name.restype = ctypes.c_char_p
        lib.fa_fwd_kernel_name.argtypes = [i, i]
        lib.fa_fwd_kernel_name.restype = ctypes.c_char_p
        lib.fa_bwd_set_phase_events.argtypes = [vp, vp, vp, vp]
        lib.fa_bwd_set_phase_events.restype = None
        lib.fa_fwd_bwd_host_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.fa_fwd_bwd_host_workspace_bytes.restype = sz
        lib.fa_unit_lists.argtypes = [i, i, i, i, i, i, vp, vp, i]
        lib.fa_unit_lists.restype = i
        lib.fa_fwd_bwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
        lib.fa_fwd_bwd_host.restype = i
        lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        lib.fa_selftest_wait_timeout.restype = i
        _lib = lib
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/fa.h declares."""
    text = open(_HEADER, encoding="utf-8").read()
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def forward_kernel_name(d: int, causal: bool) -> str:
    """Name of the kernel `forward` launches on the current device for head
    size d (fa_fwd_kernel_name)."""
    name = load_library().fa_fwd_kernel_name(int(d), int(bool(causal)))
    if name is None:
        raise RuntimeError(f"no forward kernel for d={d} on this device")
    return name.decode()


def dkdv_kernel_name(d: int, deterministic: bool = False) -> str:
    """Name of the kernel that computes dK and dV in `backward` for head size d
    (fa_bwd_dkdv_kernel_name; the deterministic form runs fa_bwd_dkdv_kernel)."""
    name = load_library().fa_bwd_dkdv_kernel_name(int(d))
    if name is None:
        raise RuntimeError(f"no dK/dV kernel for d={d}")
    return "fa_bwd_dkdv_kernel" if deterministic else name.decode()


def backward_kernel_names(d: int, deterministic: bool = False) -> tuple:
    """The three kernels `backward` launches, in order (the phases that
    set_backward_phase_events brackets)."""
    if deterministic:
        return ("fa_bwd_preprocess_kernel", "fa_bwd_dkdv_kernel", "fa_bwd_dq_kernel")
    return ("fa_bwd_preprocess_kernel", dkdv_kernel_name(d), "fa_bwd_dq_convert_kernel")


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(device: torch.device):
    """The current CUDA stream of `device` as a raw cudaStream_t."""
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(device.index))
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


class _NoSwitch:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_NO_SWITCH = _NoSwitch()


def _on(device: torch.device):
    """Make `device` current for the call (the library works on the current
    device); no switch when it already is."""
    if device.index == torch.cuda.current_device():
        return _NO_SWITCH
    return torch.cuda.device(device)


def _check_qkv(*ts: torch.Tensor):
    t0 = ts[0]
    if t0.dim() != 4:
        raise ValueError("expected tensors of shape [B, H, N, d]")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (no CPU path exists)")
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bfloat16")
        if t.shape != t0.shape or t.device != t0.device:
            raise ValueError("tensors must share shape and device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")


def _scale(scale, d):
    return 0.0 if scale is None else float(scale)


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None):
    """O, LSE = attention(q, k, v); bf16 [B,H,N,d] in, (bf16 O, fp32 LSE [B,H,N]) out."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    lib = load_library()
    with _on(q.device):
        rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, H, N, d,
                        int(bool(causal)), _scale(scale, d), _stream_handle(q.device))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd")
    return o, l


def unfused_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_fwd_unfused_workspace_bytes(B, H, N, d))


def forward_unfused(q, k, v, causal: bool = False, scale: float | None = None, workspace=None, out=None,
                    lse=None):
    """forward() the standard way: S and P materialised in HBM (fa_fwd_unfused).
    For measuring the traffic the tiled kernels avoid; same outputs."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    lib = load_library()
    nbytes = int(lib.fa_fwd_unfused_workspace_bytes(B, H, N, d))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    with _on(q.device):
        rc = lib.fa_fwd_unfused(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, H, N, d,
                                int(bool(causal)), _scale(scale, d), ws.data_ptr(), ws.numel(),
                                _stream_handle(q.device))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_unfused")
    return o, l


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_bytes(B, H, N, d))


def backward(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, workspace=None,
             dq=None, dk=None, dv=None, deterministic: bool = False):
    """dQ, dK, dV of sum(dO * O); inputs as produced by forward().

    Default (fa_bwd): one kernel forms all five products per tile and adds dQ
    partial sums into an fp32 accumulator, so dQ's last bits can vary between
    runs.  deterministic=True (fa_bwd_deterministic): a separate dQ kernel,
    bit-reproducible, slower."""
    _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous float32 [B, H, N]")
    lib = load_library()
    nbytes = int(lib.fa_bwd_workspace_bytes(B, H, N, d))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    fn = lib.fa_bwd_deterministic if deterministic else lib.fa_bwd
    with _on(q.device):
        rc = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(bool(causal)),
                _scale(scale, d), ws.data_ptr(), ws.numel(), _stream_handle(q.device))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_deterministic" if deterministic else "fa_bwd")
    return dq, dk, dv


def backward_noalloc(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, dq=None, dk=None,
                     dv=None):
    """backward(deterministic=True) without a workspace: the library's fixed
    4 MiB device array holds D (B*H*N <= NOALLOC_MAX_ROWS).  For callers that cannot allocate
    device memory; pass preallocated dq/dk/dv to allocate nothing at all.
    Calls that overlap on the GPU share the array and race."""
    _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous float32 [B, H, N]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    lib = load_library()
    with _on(q.device):
        rc = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                int(bool(causal)), _scale(scale, d), _stream_handle(q.device))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_noalloc")
    return dq, dk, dv


def host_workspace_bytes(B: int, H: int, N: int, d: int, groups: int) -> int:
    return int(load_library().fa_fwd_bwd_host_workspace_bytes(B, H, N, d, groups))


def unit_lists(kind: int, B: int, H: int, N: int, d: int, grid: int):
    """The causal kernels' per-CTA unit lists (fa_unit_lists; host only):
    kind 0 the one-SM forward, 1 the persistent backward.  Returns a list of
    `grid` lists of unit indices, or None when the shape has none (more units
    than the lists hold: the kernels deal them in serpentine order)."""
    lib = load_library()
    max_units = 4096
    start = (ctypes.c_ushort * (grid + 1))()
    order = (ctypes.c_ushort * max_units)()
    n = int(lib.fa_unit_lists(kind, B, H, N, d, grid, ctypes.cast(start, ctypes.c_void_p),
                              ctypes.cast(order, ctypes.c_void_p), max_units))
    if n < 0:
        raise FaError(n, "fa_unit_lists")
    if n == 0:
        return None
    return [list(order[start[c]:start[c + 1]]) for c in range(grid)]


def _check_host(*ts):
    t0 = ts[0]
    if t0.dim() != 4:
        raise ValueError("expected host tensors of shape [B, H, N, d]")
    for t in ts:
        if t.device.type != "cpu":
            raise ValueError("host tensors must be CPU tensors")
        if t.dtype != torch.bfloat16 or t.shape != t0.shape or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous bfloat16 of one shape")


def forward_backward_host(q, k, v, do, causal: bool = False, scale: float | None = None, groups: int = 8,
                          out=None, workspace=None, device=None):
    """O, LSE, dQ, dK, dV of attention(q, k, v) with upstream gradient dO, from
    host tensors [B, H, N, d] (bf16; page-locked for the copies to overlap) to
    host tensors, through fa_fwd_bwd_host: head groups flow through copy-in,
    kernels and copy-out at once.

    `out`: optional preallocated host (o, lse, dq, dk, dv); `workspace`:
    optional device buffer of host_workspace_bytes(B, H, N, d, groups) bytes.
    The current stream of `device` waits for the whole pipeline, so the host
    tensors hold the results once it synchronizes."""
    _check_host(q, k, v, do)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    B, H, N, d = q.shape
    if out is None:
        pin = q.is_pinned()
        mk = (lambda t: t.pin_memory()) if pin else (lambda t: t)
        out = (mk(torch.empty_like(q)), mk(torch.empty((B, H, N), dtype=torch.float32)),
               *(mk(torch.empty_like(q)) for _ in range(3)))
    o, lse, dq, dk, dv = out
    _check_host(o, dq, dk, dv)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or lse.device.type != "cpu" \
            or not lse.is_contiguous():
        raise ValueError("lse output must be a contiguous float32 CPU tensor [B, H, N]")
    lib = load_library()
    nbytes = int(lib.fa_fwd_bwd_host_workspace_bytes(B, H, N, d, groups))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if workspace is None else workspace
    with _on(dev):
        rc = lib.fa_fwd_bwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                 int(bool(causal)), _scale(scale, d), int(groups), ws.data_ptr(), ws.numel(),
                                 _stream_handle(dev))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_bwd_host")
    return o, lse, dq, dk, dv


def sync_status(device=None) -> int:
    """Synchronise the current stream and return the library's status code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(load_library().fa_sync_status(_stream_handle(dev)))


def set_backward_phase_events(events=None) -> None:
    """Record four torch.cuda.Event objects around the backward's three
    kernels (backward_kernel_names); None stops.  The events must outlive
    their use."""
    lib = load_library()
    if events is None:
        lib.fa_bwd_set_phase_events(None, None, None, None)
    else:
        for e in events:  # torch creates the CUDA event on its first record
            if e.cuda_event == 0:
                e.record()
        lib.fa_bwd_set_phase_events(*[ctypes.c_void_p(e.cuda_event) for e in events])


def last_cuda_error() -> int:
    """The cudaError_t behind the last FA_ERR_LAUNCH (fa_last_cuda_error)."""
    return int(load_library().fa_last_cuda_error())


def last_error_word() -> int:
    return int(load_library().fa_last_error_word())


def selftest_wait_timeout(limit_us: int, device=None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(load_library().fa_selftest_wait_timeout(int(limit_us), _stream_handle(dev)))


class FlashAttentionFunction(torch.autograd.Function):
    """autograd wrapper: forward and backward both run the library kernels."""

    @staticmethod
    def forward(ctx, q, k, v, causal=False, scale=None):
        o, lse = forward(q.contiguous(), k.contiguous(), v.contiguous(), causal, scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale = causal, scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, ctx.causal, ctx.scale)
        return dq, dk, dv, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None):
    return FlashAttentionFunction.apply(q, k, v, causal, scale)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
