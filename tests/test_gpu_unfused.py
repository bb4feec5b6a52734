"""GPU parity of the standard (unfused) forward, fa_fwd_unfused, against the
fp64 oracle: the comparison path of the HBM-access table in
"FlashAttention分块计算优化Transformer显存效率" (section 2.1).

It stores the scores S in fp16 (16-bit, as that table does) before the
softmax reads them back, so its LSE carries the rounding of S: a row's LSE
moves by at most max_j |dS_ij| <= 2^-11 * max_j |S_ij|.  The LSE bound used
here is therefore max(1e-3, 2^-11 * max|S|); O keeps the tiled path's bounds.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from io_aware_tiled_b200 import fa
from io_aware_tiled_b200.configs import WORKLOADS
from io_aware_tiled_b200.inputs import attention_inputs
from tests.parity import LSE_ABS, check_o, f64, max_abs

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _lse_bound(q, k, scale, rows=None):
    """max(1e-3, 2^-11 max|S|) over the given flat rows (all rows if None)."""
    qn, kn = f64(q), f64(k)
    BH, N, d = qn.shape[0] * qn.shape[1], qn.shape[2], qn.shape[3]
    qn, kn = qn.reshape(BH, N, d), kn.reshape(BH, N, d)
    smax = 0.0
    if rows is None:
        for bh in range(BH):
            smax = max(smax, float(np.abs(scale * qn[bh] @ kn[bh].T).max()))
    else:
        for r in rows:
            bh, i = divmod(int(r), N)
            smax = max(smax, float(np.abs(scale * kn[bh] @ qn[bh, i]).max()))
    return max(LSE_ABS, smax * 2.0 ** -11)


def _run(q, k, v, causal):
    dev = _dev()
    o, lse = fa.forward_unfused(q.to(dev), k.to(dev), v.to(dev), causal)
    assert fa.sync_status() == fa.FA_OK
    return o, lse


CASES = [
    # B, H, N, d, causal
    (1, 1, 1, 64, False),
    (1, 1, 1, 128, True),
    (1, 2, 17, 64, True),
    (1, 1, 128, 128, False),
    (1, 1, 129, 64, True),
    (2, 2, 300, 128, False),
    (2, 2, 300, 128, True),
    (1, 3, 640, 64, False),
    (1, 2, 1000, 128, True),
]


@pytest.mark.parametrize("B,H,N,d,causal", CASES)
def test_unfused_forward_matches_oracle(B, H, N, d, causal):
    q, k, v, _ = attention_inputs(B, H, N, d, seed=3 * N + d, with_do=False)
    scale = 1.0 / d ** 0.5
    o, lse = _run(q, k, v, causal)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), causal, scale)
    what = f"unfused {B,H,N,d,causal}"
    check_o(f64(o), ro, what)
    bound = _lse_bound(q, k, scale)
    err = max_abs(f64(lse), rl)
    assert np.isfinite(f64(lse)).all()
    assert err <= bound, f"{what}: LSE max-abs {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("causal", [False, True])
def test_unfused_at_b2h16n4096d128(causal):
    """Full size: sampled rows against the oracle, every row against the tiled
    forward (both within their bounds of the exact result)."""
    dev = _dev()
    w = WORKLOADS["fwd_b2h16n4096d128"]
    q, k, v, _ = attention_inputs(w.B, w.H, w.N, w.d, seed=w.seed, with_do=False)
    o, lse = _run(q, k, v, causal)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.arange(0, 256), rng.choice(w.B * w.H * w.N, 256, replace=False)]))
    ro, rl = oracle.forward_rows(f64(q), f64(k), f64(v), causal, w.scale, rows)
    what = f"unfused {w.name} causal={causal}"
    check_o(f64(o).reshape(-1, w.d)[rows], ro, what)
    bound = _lse_bound(q, k, w.scale, rows)
    err = max_abs(f64(lse).reshape(-1)[rows], rl)
    assert err <= bound, f"{what}: LSE max-abs {err:.3e} > {bound:.3e}"
    of, lf = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal)
    assert fa.sync_status() == fa.FA_OK
    assert float((o.float() - of.float()).abs().max()) <= 2e-2
    assert float((lse - lf).abs().max()) <= bound + LSE_ABS


def test_unfused_reuses_a_caller_workspace_and_fills_no_more_than_asked():
    """A caller-owned workspace of exactly the reported size works, twice in a
    row, and the bytes around it stay untouched."""
    dev = _dev()
    B, H, N, d = 1, 2, 200, 64
    q, k, v, _ = attention_inputs(B, H, N, d, seed=9, with_do=False)
    n = fa.unfused_workspace_bytes(B, H, N, d)
    assert n == B * H * 256 * 256 * 2
    guard = 4096
    buf = torch.full((n + 2 * guard,), 0x5A, dtype=torch.uint8, device=dev)
    ws = buf[guard:guard + n]
    outs = []
    for _ in range(2):
        o, lse = fa.forward_unfused(q.to(dev), k.to(dev), v.to(dev), True, workspace=ws)
        assert fa.sync_status() == fa.FA_OK
        outs.append((o.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert bool((buf[:guard] == 0x5A).all()) and bool((buf[guard + n:] == 0x5A).all())
    with pytest.raises(fa.FaError):
        fa.forward_unfused(q.to(dev), k.to(dev), v.to(dev), True, workspace=buf[guard:guard + n - 16])
