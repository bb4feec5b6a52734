"""Attention forward + backward on inputs in host memory, with the PCIe copies
overlapped with the kernels.

Heads are independent, so the B*H heads are split into groups that flow
through three CUDA streams: copies of group c+1 to the device, the library's
forward and backward kernels on group c, and copies of group c-1 back to the
host run at the same time (the copy engines move both directions at once).
Only copies and stream ordering happen here; every step of the attention
arithmetic runs in the library's kernels (fa.forward / fa.backward).
"""
from __future__ import annotations

import torch

from . import fa

_streams: dict = {}


def _side_streams(device: torch.device):
    key = device.index
    if key not in _streams:
        _streams[key] = tuple(torch.cuda.Stream(device=device) for _ in range(3))
    return _streams[key]


def _check_host(*ts):
    t0 = ts[0]
    if t0.dim() != 4:
        raise ValueError("expected host tensors of shape [B, H, N, d]")
    for t in ts:
        if t.device.type != "cpu" or not t.is_pinned():
            raise ValueError("host tensors must be in pinned (page-locked) CPU memory")
        if t.dtype != torch.bfloat16 or t.shape != t0.shape or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous bfloat16 of one shape")


def forward_backward_host(q, k, v, do, causal: bool = False, scale: float | None = None, groups: int = 8,
                          out=None, device=None):
    """O, LSE, dQ, dK, dV of attention(q, k, v) with upstream gradient dO,
    from pinned host tensors [B, H, N, d] (bf16) to pinned host tensors.

    `groups`: how many head groups the pipeline uses (at most B*H).  `out`:
    optional preallocated pinned (o, lse, dq, dk, dv) to fill.  Returns them
    once every copy is queued; the caller's current stream is made to wait for
    the last copy, so the host tensors hold the results after that stream
    synchronizes (torch.cuda.synchronize() or an event on it).
    """
    _check_host(q, k, v, do)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    B, H, N, d = q.shape
    BH = B * H
    if out is None:
        out = (torch.empty_like(q).pin_memory(), torch.empty((B, H, N), dtype=torch.float32).pin_memory(),
               *(torch.empty_like(q).pin_memory() for _ in range(3)))
    ho, hl, hdq, hdk, hdv = out
    _check_host(ho, hdq, hdk, hdv)
    if hl.dtype != torch.float32 or tuple(hl.shape) != (B, H, N) or not hl.is_pinned():
        raise ValueError("lse output must be pinned float32 [B, H, N]")

    per = -(-BH // max(1, min(groups, BH)))  # heads per group
    ngroups = -(-BH // per)
    cur = torch.cuda.current_stream(device)
    s_in, s_run, s_out = _side_streams(device)
    # device buffers: allocated on the current stream, which waits for every
    # side stream before this returns, so no later reuse can overtake them
    # inputs Q, K, V, dO; output O; gradients dQ, dK, dV (bf16 [B*H, N, d]); LSE
    qd, kd, vd, do_dev, o_dev, gq, gk, gv = (torch.empty((BH, N, d), dtype=torch.bfloat16, device=device)
                                             for _ in range(8))
    l_dev = torch.empty((BH, N), dtype=torch.float32, device=device)
    ws = torch.empty(fa.workspace_bytes(1, per, N, d), dtype=torch.uint8, device=device)
    flat = lambda t: t.view(BH, N, d)
    hq, hk, hv, hdo = (flat(t) for t in (q, k, v, do))
    hol, hll = flat(ho), hl.view(BH, N)
    hdql, hdkl, hdvl = flat(hdq), flat(hdk), flat(hdv)

    for s in (s_in, s_run, s_out):
        s.wait_stream(cur)
    ev_in = [torch.cuda.Event() for _ in range(ngroups)]
    ev_run = [torch.cuda.Event() for _ in range(ngroups)]
    for g in range(ngroups):
        h0, h1 = g * per, min(BH, (g + 1) * per)
        with torch.cuda.stream(s_in):
            for dst, src in ((qd, hq), (kd, hk), (vd, hv), (do_dev, hdo)):
                dst[h0:h1].copy_(src[h0:h1], non_blocking=True)
            ev_in[g].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[g])
            as4 = lambda t: t[h0:h1].view(1, h1 - h0, N, d)
            o_g, l_g = as4(o_dev), l_dev[h0:h1].view(1, h1 - h0, N)
            fa.forward(as4(qd), as4(kd), as4(vd), causal, scale, out=o_g, lse=l_g)
            fa.backward(as4(qd), as4(kd), as4(vd), o_g, as4(do_dev), l_g, causal, scale, workspace=ws,
                        dq=as4(gq), dk=as4(gk), dv=as4(gv))
            ev_run[g].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[g])
            for dst, src in ((hol, o_dev), (hll, l_dev), (hdql, gq), (hdkl, gk), (hdvl, gv)):
                dst[h0:h1].copy_(src[h0:h1], non_blocking=True)
    for s in (s_in, s_run, s_out):
        cur.wait_stream(s)
    return ho, hl, hdq, hdk, hdv
