"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(a plugin given only its input and output buffers, code under a memory pool
that must not grow).  Its D vector lives in the library's fixed device array,
and it runs the deterministic form of the backward, whose only scratch is D.

Checked through the C ABI on two calls in a row with different shapes (stale
contents of the shared array would show): bit-identical to
fa_bwd_deterministic given a workspace, and within the gradient tolerance of
fa_bwd.  One more call fills the array exactly (B*H*N = FA_NOALLOC_MAX_ROWS).
This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from io_aware_tiled_b200 import fa
from io_aware_tiled_b200.inputs import attention_inputs
from tests.parity import GRAD_REL_FROB, assert_same_up_to_summation_order, f64, rel_frob

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, k, v, o, do, lse, causal):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    rc = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal), 0.0, stream)
    return rc, (dq, dk, dv)


def test_noalloc_backward_matches_workspace_backward():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    lib = fa.load_library()
    for (B, H, N, d, causal) in [(2, 3, 1000, 128, True), (1, 4, 777, 64, False)]:
        q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=N))
        o, lse = fa.forward(q, k, v, causal)
        det = fa.backward(q, k, v, o, do, lse, causal, deterministic=True)
        fused = fa.backward(q, k, v, o, do, lse, causal)
        rc, got = _call_noalloc(lib, q, k, v, o, do, lse, causal)
        assert rc == fa.FA_OK, fa.status_string(rc)
        assert fa.sync_status(dev) == fa.FA_OK
        for name, g, r, f in zip(("dq", "dk", "dv"), got, det, fused):
            assert torch.equal(g, r), (B, H, N, d, causal, name)
            err = rel_frob(f64(g), f64(f))
            assert err <= GRAD_REL_FROB, (B, H, N, d, causal, name, err)
        assert_same_up_to_summation_order(got[0], fused[0], f"dQ {B, H, N, d} causal={causal}")


def test_noalloc_fills_its_array_exactly():
    """B*H*N = FA_NOALLOC_MAX_ROWS: the largest size the array takes; every
    row of D is used.  Still bit-identical to fa_bwd_deterministic."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    lib = fa.load_library()
    B, H, N, d = 2, 32, 16384, 64
    assert B * H * N == fa.NOALLOC_MAX_ROWS
    q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=3))
    o, lse = fa.forward(q, k, v, True)
    det = fa.backward(q, k, v, o, do, lse, True, deterministic=True)
    rc, got = _call_noalloc(lib, q, k, v, o, do, lse, True)
    assert rc == fa.FA_OK, fa.status_string(rc)
    assert fa.sync_status(dev) == fa.FA_OK
    for name, g, r in zip(("dq", "dk", "dv"), got, det):
        assert torch.equal(g, r), name


def test_noalloc_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = fa.load_library()
    rows = fa.NOALLOC_MAX_ROWS
    a = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.fa_bwd_noalloc(a, 2 * a, 3 * a, 4 * a, 5 * a, 6 * a, 7 * a, 8 * a, 9 * a, 1, 1, rows + 1, 64, 0, 0.0,
                            None)
    assert rc == fa.FA_ERR_TOO_LARGE
