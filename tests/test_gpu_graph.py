"""The library's calls can be captured in a CUDA graph and replayed: they are
asynchronous on the caller's stream, allocate nothing (given a workspace), and
bake their tensor maps into the launches' parameters.  Replays reproduce the
eager outputs exactly, except dQ of the default backward, whose partial sums
are added in an order that can vary from run to run."""
from __future__ import annotations

import pytest
import torch

from io_aware_tiled_b200 import fa
from io_aware_tiled_b200.inputs import attention_inputs
from tests.parity import assert_same_up_to_summation_order

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    B, H, N, d = 1, 4, 520, 128
    q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=5))
    o, lse = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(fa.workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)

    def step():
        fa.forward(q, k, v, True, out=o, lse=lse)
        fa.backward(q, k, v, o, do, lse, True, workspace=ws, dq=dq, dk=dk, dv=dv)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()  # first calls set the kernels' attributes outside the capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    want = [t.clone() for t in (o, lse, dq, dk, dv)]
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        step()
    for _ in range(2):
        for t in (o, lse, dq, dk, dv):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert fa.sync_status() == fa.FA_OK
        for i, (got, ref) in enumerate(zip((o, lse, dq, dk, dv), want)):
            if i == 2:  # dQ: the backward adds its partial sums in a varying order
                assert_same_up_to_summation_order(got, ref, "graph replay dQ")
            else:
                assert torch.equal(got, ref)
