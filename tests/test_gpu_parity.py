"""GPU parity: the sm_100a kernels (called through the C ABI) against the fp64 oracle.

Every input is drawn by io_aware_tiled_b200.inputs (seeded, CPU, bf16); the
oracle sees the same bf16 values widened to fp64.  Small shapes compare every
element (several tiles plus a ragged tail); the five named workloads run at
full size and compare whole heads or sampled rows the oracle computes one by
one, plus properties that hold at any size.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from io_aware_tiled_b200 import fa
from io_aware_tiled_b200.configs import WORKLOADS
from io_aware_tiled_b200.inputs import attention_inputs
from tests.parity import (assert_same_up_to_summation_order, check_grad, check_lse, check_o, f64, rel_frob,
                          to_bf16_np)

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _run_fwd(q, k, v, causal, scale=None):
    dev = _dev()
    o, lse = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal, scale)
    assert fa.sync_status() == fa.FA_OK
    return o, lse


# ---------------------------------------------------------------------------
# forward, every element, shapes spanning several tiles and ragged tails
# ---------------------------------------------------------------------------
FWD_CASES = [
    # B, H, N, d, causal, sigma_qk
    (1, 1, 256, 64, False, 1.0),
    (1, 1, 1, 64, False, 1.0),
    (1, 1, 1, 128, True, 1.0),
    (1, 2, 17, 64, True, 1.0),
    (1, 1, 127, 128, False, 1.0),
    (1, 1, 129, 128, True, 1.0),
    (2, 2, 300, 128, False, 1.0),
    (2, 2, 300, 128, True, 1.0),
    (1, 2, 640, 64, True, 1.0),      # odd number of 128-row tiles
    (1, 3, 1000, 64, True, 8.0),     # logits in the hundreds, ragged
    (1, 3, 1000, 64, False, 8.0),
    (1, 2, 777, 128, True, 2.0),
    (1, 1, 2048, 128, False, 1.0),
]


@pytest.mark.parametrize("B,H,N,d,causal,sigma", FWD_CASES)
def test_forward_matches_oracle(B, H, N, d, causal, sigma):
    q, k, v, _ = attention_inputs(B, H, N, d, seed=N + d, sigma_qk=sigma, with_do=False)
    scale = 1.0 / d ** 0.5
    o, lse = _run_fwd(q, k, v, causal)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), causal, scale)
    check_o(f64(o), ro, f"fwd {B,H,N,d,causal}")
    check_lse(f64(lse), rl, f"fwd {B,H,N,d,causal}")


def test_causal_forward_beyond_the_unit_lists():
    """Causal launches normally follow per-CTA unit lists computed on the host;
    with more than 4096 query-tile pairs (here 1200 heads x 8) the units are
    dealt in serpentine order instead.  Sampled rows of every region against
    the oracle, the first row of every head exactly V[0]."""
    dev = _dev()
    B, H, N, d = 4, 300, 2048, 64
    q, k, v, _ = attention_inputs(B, H, N, d, seed=17, with_do=False)
    o, lse = _run_fwd(q, k, v, True)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([rng.choice(B * H * N, 300, replace=False),
                                     np.arange(0, B * H * N, N) + N - 1]))
    ro, rl = oracle.forward_rows(f64(q), f64(k), f64(v), True, 1 / d ** 0.5, rows)
    check_o(f64(o).reshape(-1, d)[rows], ro, "causal, 9600 units")
    check_lse(f64(lse).reshape(-1)[rows], rl, "causal, 9600 units")
    assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0])


def test_forward_explicit_scale_and_default():
    q, k, v, _ = attention_inputs(1, 2, 200, 128, seed=5, with_do=False)
    for scale in (0.05, 0.3):
        o, lse = _run_fwd(q, k, v, True, scale)
        ro, rl = oracle.forward(f64(q), f64(k), f64(v), True, scale)
        check_o(f64(o), ro, f"scale {scale}")
        check_lse(f64(lse), rl, f"scale {scale}")
    o1, l1 = _run_fwd(q, k, v, False, None)
    o2, l2 = _run_fwd(q, k, v, False, 1.0 / 128 ** 0.5)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------------------------------------
# backward, every element
# ---------------------------------------------------------------------------
BWD_CASES = [
    (1, 1, 256, 64, False, 1.0),
    (1, 1, 1, 64, True, 1.0),
    (1, 1, 129, 128, False, 1.0),
    (1, 2, 300, 128, True, 1.0),
    (2, 1, 640, 128, True, 1.0),
    (1, 2, 1000, 64, False, 1.0),
    (1, 2, 777, 64, True, 1.0),
    (1, 1, 1024, 128, False, 1.0),
]


@pytest.mark.parametrize("deterministic", [False, True], ids=["fused", "deterministic"])
@pytest.mark.parametrize("B,H,N,d,causal,sigma", BWD_CASES)
def test_backward_matches_oracle(B, H, N, d, causal, sigma, deterministic):
    """Both backward forms: the default (five products per tile, dQ partial
    sums added into an fp32 accumulator) and the deterministic one (a
    separate dQ kernel)."""
    dev = _dev()
    q, k, v, do = attention_inputs(B, H, N, d, seed=7 * N + d, sigma_qk=sigma)
    scale = 1.0 / d ** 0.5
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, causal)
    dq, dk, dv = fa.backward(qd, kd, vd, o, dod, lse, causal, deterministic=deterministic)
    assert fa.sync_status() == fa.FA_OK
    ref = oracle.backward(f64(q), f64(k), f64(v), f64(do), causal, scale)
    what = f"bwd {B,H,N,d,causal} {'deterministic' if deterministic else 'fused'}"
    check_o(f64(o), ref["o"], what)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(f64(g), ref[name], name, what)


def _backward_vs_both_forms(q, k, v, do, dq, dk, dv, causal, scale, what, def_bound):
    """Compare gradients of every listed head with (a) the fa_bwd contract: D =
    rowsum(dO * O) over the bf16 O the backward receives (here the oracle's own
    O rounded to bf16), bound 1e-2; and (b) the definitional gradient (exact
    D = sum_j P dP), bound `def_bound`.  Returns the relative errors."""
    ref = oracle.backward(f64(q), f64(k), f64(v), f64(do), causal, scale)
    ref_c = oracle.backward(f64(q), f64(k), f64(v), f64(do), causal, scale, o_for_d=to_bf16_np(ref["o"]))
    errs = {}
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        errs[name + "_contract"] = check_grad(f64(g), ref_c[name], name, what + " (D over bf16 O)")
        errs[name + "_definitional"] = rel_frob(f64(g), ref[name])
        assert errs[name + "_definitional"] <= def_bound, (what, name, errs)
    print(what, {n: float("%.3e" % e) for n, e in errs.items()})
    return errs


def test_backward_large_logits_against_both_forms_of_D():
    """Logits in the hundreds: most rows are nearly one-hot, so dS = P (dP - D)
    is a small difference and D's rounding (O is bf16) dominates dQ and dK."""
    dev = _dev()
    B, H, N, d = 1, 2, 1000, 64
    q, k, v, do = attention_inputs(B, H, N, d, seed=11, sigma_qk=8.0)
    for causal in (False, True):
        qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
        o, lse = fa.forward(qd, kd, vd, causal)
        for det in (False, True):
            dq, dk, dv = fa.backward(qd, kd, vd, o, dod, lse, causal, deterministic=det)
            assert fa.sync_status() == fa.FA_OK
            _backward_vs_both_forms(q, k, v, do, dq, dk, dv, causal, 1.0 / 8,
                                    f"sigma 8 causal={causal} deterministic={det}", 1e-2)


# ---------------------------------------------------------------------------
# the five named workloads at full size
# ---------------------------------------------------------------------------
def _sample_rows(rng, BH, N, n):
    return np.sort(rng.choice(BH * N, size=min(n, BH * N), replace=False))


def _full_forward_check(w, causal, heads_full, n_random_rows):
    dev = _dev()
    q, k, v, do = attention_inputs(w.B, w.H, w.N, w.d, seed=w.seed, sigma_qk=w.sigma_qk, with_do=w.backward)
    o, lse = _run_fwd(q, k, v, causal)
    o_np, lse_np = f64(o).reshape(-1, w.d), f64(lse).reshape(-1)
    rng = np.random.default_rng(0)
    rows = [np.arange(h * w.N, (h + 1) * w.N) for h in heads_full]
    rows.append(_sample_rows(rng, w.B * w.H, w.N, n_random_rows))
    rows = np.unique(np.concatenate(rows))
    ro, rl = oracle.forward_rows(f64(q), f64(k), f64(v), causal, w.scale, rows)
    check_o(o_np[rows], ro, f"{w.name} causal={causal}")
    check_lse(lse_np[rows], rl, f"{w.name} causal={causal}")
    # properties at every row: finite; causal row 0 of every head is exactly V[0]
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    if causal:
        assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0])
    return q, k, v, do, o, lse


def _full_backward_check(w, causal, q, k, v, do, o, lse, heads, n_rows=0):
    """Backward at full size.  n_rows == 0: whole heads against both forms of D;
    else sampled rows of each head (the oracle computes them one by one)."""
    dev = _dev()
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    dq, dk, dv = fa.backward(qd, kd, vd, o, dod, lse, causal)
    assert fa.sync_status() == fa.FA_OK
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    def_bound = 1e-2
    if n_rows == 0:
        for bh in heads:
            b, h = divmod(bh, w.H)
            sl = lambda t: t[b:b + 1, h:h + 1]
            _backward_vs_both_forms(sl(q), sl(k), sl(v), sl(do), sl(dq).cpu(), sl(dk).cpu(), sl(dv).cpu(), causal,
                                    w.scale, f"{w.name} causal={causal} head {bh}", def_bound)
        return
    rng = np.random.default_rng(1)
    dq_np, dk_np, dv_np = (f64(t).reshape(w.B * w.H, w.N, w.d) for t in (dq, dk, dv))
    for bh in heads:
        qr = np.sort(rng.choice(w.N, size=min(n_rows, w.N), replace=False))
        kr = np.sort(rng.choice(w.N, size=min(n_rows, w.N), replace=False))
        qr[0], kr[0] = 0, w.N - 1
        ref = oracle.backward_sampled(f64(q), f64(k), f64(v), f64(do), causal, w.scale, bh, qr, kr)
        what = f"{w.name} causal={causal} head {bh}"
        check_grad(dq_np[bh][qr], ref["dq"], "dq", what)
        check_grad(dk_np[bh][kr], ref["dk"], "dk", what)
        check_grad(dv_np[bh][kr], ref["dv"], "dv", what)


def test_workload_pr1_full():
    w = WORKLOADS["pr1_b1h1n256d64"]
    q, k, v, _ = attention_inputs(w.B, w.H, w.N, w.d, seed=w.seed, with_do=False)
    o, lse = _run_fwd(q, k, v, False)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), False, w.scale)
    check_o(f64(o), ro, w.name)
    check_lse(f64(lse), rl, w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_workload_fwd_b2h16n4096d128(causal):
    w = WORKLOADS["fwd_b2h16n4096d128"]
    _full_forward_check(w, causal, heads_full=[0, 31], n_random_rows=512)


def test_workload_train_b4h32n2048d128():
    w = WORKLOADS["train_b4h32n2048d128"]
    q, k, v, do, o, lse = _full_forward_check(w, True, heads_full=[0, 127], n_random_rows=512)
    _full_backward_check(w, True, q, k, v, do, o, lse, heads=[0, 77, 127])


def test_workload_long_b1h16n16384d128():
    w = WORKLOADS["long_b1h16n16384d128"]
    q, k, v, do, o, lse = _full_forward_check(w, True, heads_full=[0], n_random_rows=384)
    _full_backward_check(w, True, q, k, v, do, o, lse, heads=[0, 15], n_rows=256)


def test_longer_than_every_workload():
    """N = 32768 (twice the long workload; 1024 query tiles of the backward, 256
    key tiles per head): the forward with and without the mask on sampled
    rows, the backward with the mask on sampled rows of both heads."""
    from io_aware_tiled_b200.configs import Workload
    w = Workload("longer_b1h2n32768d128", 1, 2, 32768, 128, (False, True), True)
    _full_forward_check(w, False, heads_full=[], n_random_rows=96)
    q, k, v, do, o, lse = _full_forward_check(w, True, heads_full=[], n_random_rows=96)
    _full_backward_check(w, True, q, k, v, do, o, lse, heads=[0, 1], n_rows=48)


@pytest.mark.parametrize("causal", [False, True])
def test_workload_ragged_b8h12n1000d64(causal):
    w = WORKLOADS["ragged_b8h12n1000d64"]
    q, k, v, do, o, lse = _full_forward_check(w, causal, heads_full=[0, 50, 95], n_random_rows=1024)
    _full_backward_check(w, causal, q, k, v, do, o, lse, heads=[0, 37, 95])


# ---------------------------------------------------------------------------
# edge cases, guard bands, determinism, autograd wrapper, errors, fault detection
# ---------------------------------------------------------------------------
def test_outputs_stay_inside_their_buffers():
    """Canary guard bands before and after O and LSE are untouched."""
    dev = _dev()
    B, H, N, d = 1, 3, 333, 128
    q, k, v, _ = attention_inputs(B, H, N, d, seed=3, with_do=False)
    guard = 4096
    n_o, n_l = B * H * N * d, B * H * N
    obuf = torch.full((n_o + 2 * guard,), -7.0, dtype=torch.bfloat16, device=dev)
    lbuf = torch.full((n_l + 2 * guard,), 123.25, dtype=torch.float32, device=dev)
    o = obuf[guard:guard + n_o].view(B, H, N, d)
    l = lbuf[guard:guard + n_l].view(B, H, N)
    fa.forward(q.to(dev), k.to(dev), v.to(dev), True, out=o, lse=l)
    assert fa.sync_status() == fa.FA_OK
    assert (obuf[:guard] == -7.0).all() and (obuf[guard + n_o:] == -7.0).all()
    assert (lbuf[:guard] == 123.25).all() and (lbuf[guard + n_l:] == 123.25).all()
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), True, 1 / d ** 0.5)
    check_o(f64(o), ro, "guarded")


def test_gradient_outputs_stay_inside_their_buffers():
    dev = _dev()
    B, H, N, d = 1, 2, 200, 64
    q, k, v, do = attention_inputs(B, H, N, d, seed=4)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, False)
    guard, n = 2048, B * H * N * d
    bufs = [torch.full((n + 2 * guard,), 3.5, dtype=torch.bfloat16, device=dev) for _ in range(3)]
    views = [b[guard:guard + n].view(B, H, N, d) for b in bufs]
    fa.backward(qd, kd, vd, o, dod, lse, False, dq=views[0], dk=views[1], dv=views[2])
    assert fa.sync_status() == fa.FA_OK
    for b in bufs:
        assert (b[:guard] == 3.5).all() and (b[guard + n:] == 3.5).all()


def test_outputs_at_a_16_byte_offset():
    """O, dK and dV are written with 32-byte stores when the row start is
    32-byte aligned and with 16-byte stores otherwise (the ABI asks for 16-byte
    alignment).  Outputs 8 elements (16 bytes) past a 32-byte boundary equal,
    bit for bit, those written into aligned buffers, for every forward kernel
    and the backward, and the guard elements around them stay untouched."""
    dev = _dev()
    for B, H, N, d, causal in ((1, 2, 300, 128, False), (1, 2, 300, 128, True), (1, 2, 300, 64, False)):
        q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=41))
        n = B * H * N * d
        o_ref, lse = fa.forward(q, k, v, causal)
        obuf = torch.full((n + 64,), -7.0, dtype=torch.bfloat16, device=dev)
        o = obuf[8:8 + n].view(B, H, N, d)
        assert o.data_ptr() % 32 == 16
        fa.forward(q, k, v, causal, out=o, lse=torch.empty_like(lse))
        assert fa.sync_status() == fa.FA_OK
        assert torch.equal(o, o_ref), (B, H, N, d, causal)
        assert (obuf[:8] == -7.0).all() and (obuf[8 + n:] == -7.0).all()
        g_ref = fa.backward(q, k, v, o_ref, do, lse, causal)
        bufs = [torch.full((n + 64,), 3.5, dtype=torch.bfloat16, device=dev) for _ in range(3)]
        views = [b[8:8 + n].view(B, H, N, d) for b in bufs]
        fa.backward(q, k, v, o_ref, do, lse, causal, dq=views[0], dk=views[1], dv=views[2])
        assert fa.sync_status() == fa.FA_OK
        assert torch.equal(views[1], g_ref[1]) and torch.equal(views[2], g_ref[2])
        assert_same_up_to_summation_order(views[0], g_ref[0], "dQ at a 16-byte offset")
        for b in bufs:
            assert (b[:8] == 3.5).all() and (b[8 + n:] == 3.5).all()


def test_forward_and_backward_are_deterministic():
    """The forward and the deterministic backward give identical bits on
    repeated calls.  The default backward gives identical dK and dV; its dQ
    partial sums reach the accumulator in a varying order, so dQ agrees up to
    that order."""
    dev = _dev()
    q, k, v, do = attention_inputs(1, 4, 1000, 128, seed=9)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    for causal in (False, True):
        o1, l1 = fa.forward(qd, kd, vd, causal)
        o2, l2 = fa.forward(qd, kd, vd, causal)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        g1 = fa.backward(qd, kd, vd, o1, dod, l1, causal, deterministic=True)
        g2 = fa.backward(qd, kd, vd, o1, dod, l1, causal, deterministic=True)
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)
        f1 = fa.backward(qd, kd, vd, o1, dod, l1, causal)
        f2 = fa.backward(qd, kd, vd, o1, dod, l1, causal)
        assert torch.equal(f1[1], f2[1]) and torch.equal(f1[2], f2[2])
        assert_same_up_to_summation_order(f1[0], f2[0], f"dQ causal={causal}")


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 1000, 128), (2, 3, 300, 64), (1, 1, 129, 128), (1, 2, 2048, 64),
                                     (1, 1, 1, 128)])
def test_fused_and_deterministic_backward_agree(B, H, N, d):
    """The two backward forms form dK and dV from the same products.  With the
    mask both walk the query tiles in the same order, so dK and dV are
    bit-identical; without it the fused kernel starts each key tile at a
    different query tile (spreading the dQ additions over the accumulator),
    which changes only the summation order.  dQ agrees up to summation order
    in both cases."""
    dev = _dev()
    q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=13 * N + d))
    for causal in (False, True):
        o, lse = fa.forward(q, k, v, causal)
        fu = fa.backward(q, k, v, o, do, lse, causal)
        de = fa.backward(q, k, v, o, do, lse, causal, deterministic=True)
        assert fa.sync_status() == fa.FA_OK
        what = f"{B,H,N,d} causal={causal}"
        assert_same_up_to_summation_order(fu[0], de[0], "dQ " + what)
        for name, a, b in (("dK", fu[1], de[1]), ("dV", fu[2], de[2])):
            if causal:
                assert torch.equal(a, b), name + " " + what
            else:
                assert_same_up_to_summation_order(a, b, name + " " + what)


def test_persistent_backward_walks_every_unit():
    """The default backward's kernel is persistent: one CTA per SM walks its
    key-tile units (lists computed on the host with the mask, at most 4096
    units; beyond that, and without the mask, a serpentine deal).  Shapes
    with one unit per CTA, many units per CTA and more units than the lists
    hold all give the deterministic form's dK and dV bit for bit with the mask
    (the same products in the same order) and dQ up to summation order."""
    dev = _dev()
    for B, H, N, d, causals in ((1, 1, 130, 64, (False, True)),        # 2 units, fewer than the SMs
                                (2, 8, 1280, 128, (False, True)),      # 160 units: some CTAs take two
                                (4, 300, 1024, 64, (True,))):          # 9600 units: past the lists
        q, k, v, do = (t.to(dev) for t in attention_inputs(B, H, N, d, seed=31 + N))
        for causal in causals:
            o, lse = fa.forward(q, k, v, causal)
            fu = fa.backward(q, k, v, o, do, lse, causal)
            de = fa.backward(q, k, v, o, do, lse, causal, deterministic=True)
            assert fa.sync_status() == fa.FA_OK
            what = f"{B,H,N,d} causal={causal}"
            assert_same_up_to_summation_order(fu[0], de[0], "dQ " + what)
            for name, a, b in (("dK", fu[1], de[1]), ("dV", fu[2], de[2])):
                if causal:
                    assert torch.equal(a, b), name + " " + what
                else:
                    assert_same_up_to_summation_order(a, b, name + " " + what)


def test_autograd_wrapper_runs_library_kernels():
    dev = _dev()
    q, k, v, do = attention_inputs(1, 2, 256, 64, seed=12)
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    o = fa.attention(qd, kd, vd, True)
    o.backward(do.to(dev))
    o2, lse = fa.forward(qd.detach(), kd.detach(), vd.detach(), True)
    g = fa.backward(qd.detach(), kd.detach(), vd.detach(), o2, do.to(dev), lse, True)
    assert torch.equal(o.detach(), o2)
    assert_same_up_to_summation_order(qd.grad, g[0], "autograd dQ")
    for t, ref in zip((kd, vd), g[1:]):
        assert torch.equal(t.grad, ref)


def test_invalid_arguments_on_gpu():
    dev = _dev()
    q = torch.zeros(1, 1, 64, 96, dtype=torch.bfloat16, device=dev)
    with pytest.raises(fa.FaError) as e:
        fa.forward(q, q.clone(), q.clone())
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError):
        fa.forward(q, q.float(), q)


def test_wait_timeout_is_reported_and_context_survives():
    """A wait on a barrier nothing signals runs out after 2 ms; the library
    reports FA_ERR_TIMEOUT and the next launches work normally."""
    dev = _dev()
    assert fa.selftest_wait_timeout(2000) == fa.FA_OK
    assert fa.sync_status() == fa.FA_ERR_TIMEOUT
    assert fa.last_error_word() == (255 << 8) | 1
    assert fa.sync_status() == fa.FA_OK  # cleared
    q, k, v, _ = attention_inputs(1, 1, 256, 64, seed=0, with_do=False)
    o, lse = _run_fwd(q, k, v, False)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), False, 1 / 8)
    check_o(f64(o), ro, "after timeout")


PAIR_CASES = [(1, 3, 1000, True), (1, 3, 1000, False), (2, 2, 300, True), (1, 3, 333, True),
              (1, 1, 129, False), (1, 1, 1, True), (1, 2, 2048, False), (1, 1, 640, True)]


@pytest.mark.parametrize("B,H,N,causal", PAIR_CASES)
def test_both_forward_kernels_for_d128(B, H, N, causal, monkeypatch):
    """d = 128 has two forward kernels: one SM per CTA, and CTA pairs (2-SM
    MMAs).  FA_FWD_PAIR=0 / =1 forces either; both match the oracle, ragged
    tails and query tiles past N included."""
    d = 128
    q, k, v, _ = attention_inputs(B, H, N, d, seed=21 + N, with_do=False)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), causal, 1 / d ** 0.5)
    for mode in ("0", "1"):
        monkeypatch.setenv("FA_FWD_PAIR", mode)
        o, lse = _run_fwd(q, k, v, causal)
        what = f"{'paired' if mode == '1' else 'one-SM'} {B,H,N} causal={causal}"
        check_o(f64(o), ro, what)
        check_lse(f64(lse), rl, what)
    monkeypatch.delenv("FA_FWD_PAIR")


def test_paired_forward_walks_every_unit_with_the_mask(monkeypatch):
    """With the mask the paired kernel follows per-pair unit lists (at most
    4096 units; beyond, a serpentine deal).  Shapes with several units per
    CTA pair, on the lists and past them: sampled heads, from both ends of
    every batch, match the oracle; every head's LSE matches the one-SM
    kernel's to rounding, so no unit was skipped or run twice."""
    dev = _dev()
    monkeypatch.setenv("FA_FWD_PAIR", "1")
    assert fa.forward_kernel_name(128, True) == "fa_fwd_2sm_kernel"
    d = 128
    for B, H, N in ((2, 40, 1000), (4, 300, 2048)):   # 320 units on the lists; 9600, past them
        q, k, v, _ = attention_inputs(B, H, N, d, seed=51 + N, with_do=False)
        qd, kd, vd = (t.to(dev) for t in (q, k, v))
        o, lse = fa.forward(qd, kd, vd, True)
        assert fa.sync_status() == fa.FA_OK
        monkeypatch.setenv("FA_FWD_PAIR", "0")
        _, lse1 = fa.forward(qd, kd, vd, True)
        assert fa.sync_status() == fa.FA_OK
        monkeypatch.setenv("FA_FWD_PAIR", "1")
        assert (lse - lse1).abs().max().item() <= 1e-3, f"{B,H,N} LSE of the two kernels"
        for b, h in ((0, 0), (B - 1, H - 1), (B // 2, H // 2)):
            ro, rl = oracle.forward(f64(q[b:b + 1, h:h + 1]), f64(k[b:b + 1, h:h + 1]), f64(v[b:b + 1, h:h + 1]),
                                    True, 1 / d ** 0.5)
            what = f"paired {B,H,N} causal head {b},{h}"
            check_o(f64(o[b:b + 1, h:h + 1].cpu()), ro, what)
            check_lse(f64(lse[b:b + 1, h:h + 1].cpu()), rl, what)
        del qd, kd, vd, o, lse, lse1
    monkeypatch.delenv("FA_FWD_PAIR")


def test_forward_kernel_name_follows_the_routing(monkeypatch):
    """fa_fwd_kernel_name reports the kernel fa_fwd launches: CTA pairs for
    d = 128 without the mask, one SM per CTA otherwise, FA_FWD_PAIR forcing
    either for d = 128; no name for an unsupported head size."""
    monkeypatch.delenv("FA_FWD_PAIR", raising=False)
    assert fa.forward_kernel_name(128, False) == "fa_fwd_2sm_kernel"
    assert fa.forward_kernel_name(128, True) == "fa_fwd_kernel"
    assert fa.forward_kernel_name(64, False) == "fa_fwd_kernel"
    assert fa.forward_kernel_name(64, True) == "fa_fwd_kernel"
    monkeypatch.setenv("FA_FWD_PAIR", "0")
    assert fa.forward_kernel_name(128, False) == "fa_fwd_kernel"
    monkeypatch.setenv("FA_FWD_PAIR", "1")
    assert fa.forward_kernel_name(128, True) == "fa_fwd_2sm_kernel"
    assert fa.forward_kernel_name(64, True) == "fa_fwd_kernel"
    with pytest.raises(RuntimeError):
        fa.forward_kernel_name(96, False)


BN64_CASES = [(1, 2, 1000, 128, True), (1, 2, 1000, 128, False), (1, 1, 129, 64, True), (2, 2, 300, 64, False),
              (1, 1, 1, 128, True), (1, 3, 640, 128, True), (1, 1, 200, 64, True)]


@pytest.mark.parametrize("B,H,N,d,causal", BN64_CASES)
def test_forward_with_64_key_tiles(B, H, N, d, causal, monkeypatch):
    """FA_FWD_BN=64 runs the one-SM kernel with 64-key K/V tiles (tile-size
    comparisons): two key tiles per query tile's width, so the causal
    diagonal spans two tiles and the second may be fully masked for half the
    rows."""
    q, k, v, _ = attention_inputs(B, H, N, d, seed=31 + N + d, with_do=False)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), causal, 1 / d ** 0.5)
    monkeypatch.setenv("FA_FWD_BN", "64")
    assert fa.forward_kernel_name(d, causal) == "fa_fwd_kernel"
    o, lse = _run_fwd(q, k, v, causal)
    monkeypatch.delenv("FA_FWD_BN")
    what = f"64-key tiles {B,H,N,d} causal={causal}"
    check_o(f64(o), ro, what)
    check_lse(f64(lse), rl, what)


@pytest.mark.parametrize("threshold", ["0", "3", "16", "30"])
@pytest.mark.parametrize("pair", ["0", "1"])
def test_forward_rescale_threshold(threshold, pair, monkeypatch):
    """FA_FWD_RESCALE sets how far a row maximum may grow before O is
    rescaled (0: on every growth).  Logits in the hundreds (sigma 8) make the
    maxima jump across tiles, so rescaling happens often; every threshold
    gives the oracle's O and LSE."""
    B, H, N, d = 1, 2, 777, 128
    q, k, v, _ = attention_inputs(B, H, N, d, seed=41, sigma_qk=8.0, with_do=False)
    ro, rl = oracle.forward(f64(q), f64(k), f64(v), True, 1 / d ** 0.5)
    ro2, rl2 = oracle.forward(f64(q), f64(k), f64(v), False, 1 / d ** 0.5)
    monkeypatch.setenv("FA_FWD_RESCALE", threshold)
    monkeypatch.setenv("FA_FWD_PAIR", pair)
    for causal, (o_ref, l_ref) in ((True, (ro, rl)), (False, (ro2, rl2))):
        o, lse = _run_fwd(q, k, v, causal)
        what = f"rescale threshold {threshold} pair={pair} causal={causal}"
        check_o(f64(o), o_ref, what)
        check_lse(f64(lse), l_ref, what)


def test_host_pipeline_equals_the_device_path():
    """fa_fwd_bwd_host (host tensors in and out, head groups through copy-in,
    kernels and copy-out on the library's streams) returns the device path's
    outputs: the same kernels on the same heads; only dQ's partial sums may
    be added in another order.  Page-locked and ordinary host memory alike."""
    from io_aware_tiled_b200.host_pipeline import forward_backward_host
    dev = _dev()
    B, H, N, d = 2, 3, 300, 128
    q, k, v, do = attention_inputs(B, H, N, d, seed=77)
    for causal in (False, True):
        o, lse = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal)
        g = fa.backward(q.to(dev), k.to(dev), v.to(dev), o, do.to(dev), lse, causal)
        for pinned, groups in ((True, 4), (False, 1), (True, 6), (True, 100)):
            ins = [t.pin_memory() if pinned else t for t in (q, k, v, do)]
            host = forward_backward_host(*ins, causal, groups=groups, device=dev)
            torch.cuda.synchronize()
            assert fa.sync_status() == fa.FA_OK
            for i, (got, want) in enumerate(zip(host, (o, lse, *g))):
                what = f"host pipeline causal={causal} pinned={pinned} groups={groups} output {i}"
                if i == 2:  # dQ: partial sums added in a varying order
                    assert_same_up_to_summation_order(got, want, what)
                else:
                    assert torch.equal(got, want.cpu()), what
    # 16 heads in four groups of 4: more groups than the pipeline's three slots
    B, H, N, d = 2, 8, 200, 64
    q, k, v, do = attention_inputs(B, H, N, d, seed=78)
    for causal in (False, True):
        o, lse = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal)
        g = fa.backward(q.to(dev), k.to(dev), v.to(dev), o, do.to(dev), lse, causal)
        host = forward_backward_host(*(t.pin_memory() for t in (q, k, v, do)), causal, groups=4, device=dev)
        torch.cuda.synchronize()
        assert fa.sync_status() == fa.FA_OK
        for i, (got, want) in enumerate(zip(host, (o, lse, *g))):
            what = f"host pipeline 16 heads causal={causal} output {i}"
            if i == 2:
                assert_same_up_to_summation_order(got, want, what)
            else:
                assert torch.equal(got, want.cpu()), what
    with pytest.raises(ValueError):
        forward_backward_host(q.to(dev), k, v, do)  # a device tensor where host memory is expected
