"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each expected value comes from
the pages' worked example, a closed form, an invariant, an independent
algorithm written here (the online-softmax merge), brute force, finite
differences, or a library routine (torch CPU fp64 as a special case).
"""
from __future__ import annotations

import math
import os
import random

import numpy as np
import pytest
import torch

import oracle
from oracle.capacity import attention_score_bytes
from io_aware_tiled_b200.inputs import attention_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape) * scale


# --------------------------------------------------------------------------
# worked example: blockwise softmax of [1, 2, 3, 4] ("图解Flash Attention运算原理",
# section "Softmax 的分块计算")
# --------------------------------------------------------------------------

def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(r) for r in rest]
    return vals


def test_worked_example_blockwise_softmax():
    g = _read_golden("blockwise_softmax_1234.txt")
    x, b0, b1 = g["x"], g["block0"], g["block1"]
    # the page's local statistics
    assert [max(b0), max(b1)] == g["local_max"]
    assert max(x) == g["global_max"][0]
    num0 = sum(math.exp(t - max(b0)) for t in b0)
    num1 = sum(math.exp(t - max(b1)) for t in b1)
    assert num0 == pytest.approx(math.exp(-1) + 1, rel=1e-15)
    assert num1 == pytest.approx(math.exp(-1) + 1, rel=1e-15)
    # merge: block 0 scaled by e^{2-4}
    factor = math.exp(g["merge_exponent_block0"][0])
    assert factor == pytest.approx(math.exp(max(b0) - max(x)), rel=1e-15)
    merged = num0 * factor + num1
    assert merged == pytest.approx((1 + math.exp(-1)) * (1 + math.exp(-2)), rel=1e-15)
    expected = [math.exp(t - max(x)) / merged for t in x]
    expected_lse = max(x) + math.log(merged)
    # The oracle sees the same row as scores: d=4, q0 = e_0, k_j = (x_j, 0, 0, 0), scale 1,
    # V = identity so that O row 0 is the probability row itself.
    N = d = 4
    q = np.zeros((1, 1, N, d)); q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, N, d)); k[0, 0, :, 0] = x
    v = np.eye(N)[None, None]
    o, lse = oracle.forward(q, k, v, causal=False, scale=1.0)
    np.testing.assert_allclose(o[0, 0, 0], expected, rtol=1e-15, atol=1e-16)
    assert lse[0, 0, 0] == pytest.approx(expected_lse, rel=1e-15)
    p = oracle.probs(q, k, causal=False, scale=1.0)
    np.testing.assert_allclose(p[0], expected, rtol=1e-15, atol=1e-16)
    # the numbers quoted for this example
    np.testing.assert_allclose(expected, [0.0320586, 0.0871443, 0.2368828, 0.6439143], atol=5e-8)
    assert expected_lse == pytest.approx(4.4401897, abs=5e-8)


# --------------------------------------------------------------------------
# online softmax ("FlashAttention分块计算优化Transformer显存效率", section 3.2): an
# independent implementation here, over random splits, must equal the oracle's one pass
# --------------------------------------------------------------------------

def _online_attention_row(s_row, v, splits):
    """Running max, running sum and running output over blocks of keys, then O / l."""
    m, l, out = -math.inf, 0.0, np.zeros(v.shape[1])
    start = 0
    for stop in list(splits) + [len(s_row)]:
        blk = s_row[start:stop]
        if len(blk) == 0:
            continue
        m_new = max(m, float(np.max(blk)))
        corr = math.exp(m - m_new) if m != -math.inf else 0.0
        p = np.exp(blk - m_new)
        l = l * corr + float(p.sum())
        out = out * corr + p @ v[start:stop]
        m = m_new
        start = stop
    return out / l, m + math.log(l)


@pytest.mark.parametrize("causal", [False, True])
def test_online_merge_any_split_equals_one_pass(causal):
    rnd = random.Random(7)
    B, H, N, d = 1, 2, 37, 5
    q, k, v = _rand((B, H, N, d), 1), _rand((B, H, N, d), 2), _rand((B, H, N, d), 3)
    scale = 0.61
    o, lse = oracle.forward(q, k, v, causal, scale)
    for h in range(H):
        s = (q[0, h] @ k[0, h].T) * scale
        for i in range(N):
            row = s[i].copy()
            if causal:
                row = row[: i + 1]
            vv = v[0, h][: len(row)]
            splits = sorted(rnd.sample(range(1, len(row)), min(3, len(row) - 1))) if len(row) > 1 else []
            oi, li = _online_attention_row(row, vv, splits)
            np.testing.assert_allclose(o[0, h, i], oi, rtol=1e-12, atol=1e-13)
            assert lse[0, h, i] == pytest.approx(li, rel=1e-13, abs=1e-13)


# --------------------------------------------------------------------------
# invariants and closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k = _rand((2, 3, 29, 8), 4, 3.0), _rand((2, 3, 29, 8), 5, 3.0)
    for bh in (0, 4):
        p = oracle.probs(q, k, causal, 0.35, bh=bh)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        assert (p >= 0).all()
        if causal:
            assert np.all(np.triu(p, 1) == 0.0)


def test_causal_row_zero_returns_v0():
    q, k, v = _rand((2, 2, 19, 16), 6), _rand((2, 2, 19, 16), 7), _rand((2, 2, 19, 16), 8)
    scale = 0.25
    o, lse = oracle.forward(q, k, v, True, scale)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * np.einsum("bhc,bhc->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=1e-14, atol=1e-15)


def test_zero_scores_give_means():
    B, H, N, d = 1, 2, 23, 4
    k, v = _rand((B, H, N, d), 9), _rand((B, H, N, d), 10)
    q = np.zeros((B, H, N, d))
    o, lse = oracle.forward(q, k, v, False, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), rtol=1e-13,
                               atol=1e-14)
    np.testing.assert_allclose(lse, math.log(N), rtol=1e-15)
    o, lse = oracle.forward(q, k, v, True, 0.5)
    prefix = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, N + 1))[None, None, :].repeat(H, 1),
                               rtol=1e-14, atol=1e-15)
    # scale = 0 has the same effect as Q = 0
    o2, lse2 = oracle.forward(_rand((B, H, N, d), 11), k, v, False, 0.0)
    np.testing.assert_allclose(o2, np.broadcast_to(v.mean(axis=2, keepdims=True), o2.shape), rtol=1e-13,
                               atol=1e-14)


def test_key_permutation_invariance_noncausal():
    B, H, N, d = 1, 1, 31, 6
    q, k, v = _rand((B, H, N, d), 12), _rand((B, H, N, d), 13), _rand((B, H, N, d), 14)
    perm = np.random.default_rng(0).permutation(N)
    o1, l1 = oracle.forward(q, k, v, False, 0.4)
    o2, l2 = oracle.forward(q, k[:, :, perm], v[:, :, perm], False, 0.4)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_fp64(causal):
    B, H, N, d = 2, 2, 45, 16
    q, k, v = _rand((B, H, N, d), 15, 2.0), _rand((B, H, N, d), 16, 2.0), _rand((B, H, N, d), 17)
    scale = 1 / math.sqrt(d)
    o, lse = oracle.forward(q, k, v, causal, scale)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    s = (tq @ tk.transpose(-1, -2)) * scale
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    ref = torch.softmax(s, dim=-1) @ tv
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-13, atol=1e-13)


def test_brute_force_tiny():
    """Pure-Python loops from the definition, N <= 8, d <= 4."""
    rng = random.Random(3)
    for N, d, causal in [(1, 1, False), (3, 2, True), (5, 4, False), (8, 3, True), (8, 4, False)]:
        q = [[rng.gauss(0, 1) for _ in range(d)] for _ in range(N)]
        k = [[rng.gauss(0, 1) for _ in range(d)] for _ in range(N)]
        v = [[rng.gauss(0, 1) for _ in range(d)] for _ in range(N)]
        scale = 0.8
        exp_o, exp_l = [], []
        for i in range(N):
            s = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(N)]
            if causal:
                s = [s[j] if j <= i else -math.inf for j in range(N)]
            m = max(s)
            z = sum(math.exp(t - m) for t in s)
            exp_o.append([sum(math.exp(s[j] - m) / z * v[j][c] for j in range(N)) for c in range(d)])
            exp_l.append(m + math.log(z))
        o, lse = oracle.forward(np.array(q)[None, None], np.array(k)[None, None],
                                np.array(v)[None, None], causal, scale)
        np.testing.assert_allclose(o[0, 0], exp_o, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0], exp_l, rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------
# backward: finite differences, autograd, the two forms of D, row sums of dS
# --------------------------------------------------------------------------

def _loss(q, k, v, do, causal, scale):
    o, _ = oracle.forward(q, k, v, causal, scale)
    return float((o * do).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_central_differences(causal):
    B, H, N, d = 1, 2, 7, 3
    q, k, v, do = (_rand((B, H, N, d), s) for s in (20, 21, 22, 23))
    scale = 0.9
    g = oracle.backward(q, k, v, do, causal, scale)
    eps = 1e-5
    for name, x, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            fd[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, causal, scale)
                       - _loss(args_m["q"], args_m["k"], args_m["v"], do, causal, scale)) / (2 * eps)
        err = np.linalg.norm(fd - grad) / max(np.linalg.norm(fd), 1e-30)
        assert err < 1e-7, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd(causal):
    B, H, N, d = 2, 2, 33, 8
    q, k, v, do = (_rand((B, H, N, d), s, 1.5) for s in (30, 31, 32, 33))
    scale = 1 / math.sqrt(d)
    g = oracle.backward(q, k, v, do, causal, scale)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    s = (tq @ tk.transpose(-1, -2)) * scale
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.from_numpy(do))
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g["o"], o.detach().numpy(), rtol=1e-12, atol=1e-13)


def test_two_forms_of_D_agree():
    q, k, v, do = (_rand((1, 3, 50, 16), s) for s in (40, 41, 42, 43))
    for causal in (False, True):
        g = oracle.backward(q, k, v, do, causal, 0.3)
        np.testing.assert_allclose(g["D"], g["D_rowsum"], rtol=1e-12, atol=1e-13)
        # passing the oracle's own O as the O for D reproduces the definitional gradients
        g2 = oracle.backward(q, k, v, do, causal, 0.3, o_for_d=g["o"])
        for n in ("dq", "dk", "dv"):
            np.testing.assert_allclose(g2[n], g[n], rtol=1e-10, atol=1e-12)


def test_dS_rows_sum_to_zero():
    """sum_j dS_ij = 0 for every row, so with all key rows equal dQ vanishes."""
    B, H, N, d = 1, 1, 17, 4
    q, v, do = (_rand((B, H, N, d), s) for s in (50, 51, 52))
    k = np.broadcast_to(_rand((1, 1, 1, d), 53), (B, H, N, d)).copy()
    for causal in (False, True):
        g = oracle.backward(q, k, v, do, causal, 0.7)
        assert np.abs(g["dq"]).max() < 1e-13
        assert np.abs(g["dk"]).max() > 1e-3  # the key gradients do not vanish


# --------------------------------------------------------------------------
# the sampled entry points agree with the full ones
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_forward_rows_match_full(causal):
    B, H, N, d = 2, 2, 40, 8
    q, k, v = (_rand((B, H, N, d), s) for s in (60, 61, 62))
    o, lse = oracle.forward(q, k, v, causal, 0.4)
    rows = np.array([0, 5, 39, 40, 77, 159])
    orow, lrow = oracle.forward_rows(q, k, v, causal, 0.4, rows)
    np.testing.assert_allclose(orow, o.reshape(-1, d)[rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lrow, lse.reshape(-1)[rows], rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_sampled_matches_full(causal):
    B, H, N, d = 1, 3, 45, 8
    q, k, v, do = (_rand((B, H, N, d), s) for s in (70, 71, 72, 73))
    g = oracle.backward(q, k, v, do, causal, 0.45)
    for bh in (0, 2):
        qr, kr = [0, 7, 44], [0, 13, 44]
        s = oracle.backward_sampled(q, k, v, do, causal, 0.45, bh, qr, kr)
        np.testing.assert_allclose(s["dq"], g["dq"][0, bh][qr], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(s["dk"], g["dk"][0, bh][kr], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(s["dv"], g["dv"][0, bh][kr], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(s["lse"], g["lse"][0, bh], rtol=1e-14)
        np.testing.assert_allclose(s["D"], g["D"][0, bh], rtol=1e-11, atol=1e-13)
        s2 = oracle.backward_sampled(q, k, v, do, causal, 0.45, bh, qr, kr, o_for_d=g["o"])
        np.testing.assert_allclose(s2["D"], g["D_rowsum"][0, bh], rtol=1e-11, atol=1e-13)


def test_oracle_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.forward(np.zeros((1, 1, 0, 4)), np.zeros((1, 1, 0, 4)), np.zeros((1, 1, 0, 4)), False, 1.0)
    with pytest.raises(ValueError):
        oracle.forward_rows(np.zeros((1, 1, 4, 4)), np.zeros((1, 1, 4, 4)), np.zeros((1, 1, 4, 4)),
                            False, 1.0, [4])


# --------------------------------------------------------------------------
# capacity statement and the input recipe
# --------------------------------------------------------------------------

def test_score_bytes_of_long_sequence_workload():
    """The long-sequence workload's materialised S (B=1, H=16, N=16384, bf16) is 8 GiB
    ("14. FlashAttention Memory Model", Q1 check)."""
    assert attention_score_bytes(16384, 1, 16, 2) == 8 * 2 ** 30
    assert attention_score_bytes(4096) == 32 * 2 ** 20
    with pytest.raises(ValueError):
        attention_score_bytes(0)


def test_input_recipe_is_seeded_and_bf16():
    a = attention_inputs(1, 2, 33, 64, seed=0, sigma_qk=8.0)
    b = attention_inputs(1, 2, 33, 64, seed=0, sigma_qk=8.0)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 2, 33, 64) and x.is_contiguous()
        assert torch.equal(x, y)
    c = attention_inputs(1, 2, 33, 64, seed=1)
    assert not torch.equal(a[2], c[2])
    # sigma multiplies Q and K only
    assert 5.0 < float(a[0].float().std()) < 11.0 and 0.7 < float(a[2].float().std()) < 1.3
    with pytest.raises(ValueError):
        attention_inputs(1, 1, 0, 64)


def test_parity_helpers_format_floor():
    """The O check's format floor: half a bf16 spacing, e.g. 1/128 on [2, 4)."""
    from tests.parity import half_ulp_bf16, o_excess_error
    np.testing.assert_array_equal(half_ulp_bf16([1.0, 1.5, 2.0, 3.9, 0.25]),
                                  [2 ** -8, 2 ** -8, 2 ** -7, 2 ** -7, 2 ** -10])
    # a one-spacing flip next to a midpoint is within the budget, an error of 0.02 is not
    assert o_excess_error([3.0 + 2 ** -6], [3.0 + 2 ** -7 + 1e-6]) < 1e-2
    assert o_excess_error([3.02], [3.0]) > 1e-2
