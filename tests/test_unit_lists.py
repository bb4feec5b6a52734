"""The causal kernels' per-CTA unit lists (host logic, no GPU): every unit
exactly once, each CTA's units in the kernel's order, and the longest-
processing-time assignment's balance over the SMs."""
from __future__ import annotations

import pytest

from io_aware_tiled_b200 import fa

EINVAL = -1
SMS = 148
FWD_GROUP_BYTES = 32 << 20  # K and V of a head group kept in L2: the forward's lists
BWD_GROUP_BYTES = 32 << 20  # and the backward's


def _group(BH, N, d, group_bytes):
    g = group_bytes // (4 * N * d)
    return BH if g >= BH else max(1, g)


def _fwd_units(BH, N):
    """Forward unit u = r*BH + bh: query-tile pair NP-1-r of head bh; cost in
    128-key steps: the pair's two tiles' key tiles plus two."""
    NQT, NKT = -(-N // 128), -(-N // 128)
    NP = (NQT + 1) // 2
    cost = {}
    for u in range(BH * NP):
        qp = NP - 1 - u // BH
        cost[u] = min(2 * qp + 1, NKT) + min(2 * qp + 2, NKT) + 2
    return cost


def _fwd_position(BH, N, d):
    """Position of each forward unit in the assignment order: head groups,
    longest pairs first inside a group."""
    NP = (-(-N // 128) + 1) // 2
    G = _group(BH, N, d, FWD_GROUP_BYTES)
    pos, p = {}, 0
    for g0 in range(0, BH, G):
        for r in range(NP):
            for bh in range(g0, min(BH, g0 + G)):
                pos[r * BH + bh] = p
                p += 1
    return pos


def _bwd_units(BH, N, d):
    """Backward unit u (grouped longest-first numbering) -> key tile kt; cost
    = the query tiles of 64 rows that see the key tile, plus one."""
    NKT, NQT = -(-N // 128), -(-N // 64)
    G = _group(BH, N, d, BWD_GROUP_BYTES)
    cost = {}
    for u in range(BH * NKT):
        g, v = divmod(u, G * NKT)
        gh = min(G, BH - g * G)
        kt = v // gh
        cost[u] = NQT - 2 * kt + 1
    return cost


def _check(lists, cost, order_pos, grid):
    """Each unit once, in the kernel's order within a CTA; the busiest CTA
    within one unit of the mean (the list-scheduling bound)."""
    assert len(lists) == grid
    flat = [u for L in lists for u in L]
    assert sorted(flat) == sorted(cost), "every unit exactly once"
    for L in lists:
        assert all(order_pos[a] < order_pos[b] for a, b in zip(L, L[1:])), "a CTA's units in the kernel's order"
    loads = [sum(cost[u] for u in L) for L in lists]
    mean = sum(loads) / grid
    assert max(loads) <= mean + max(cost.values()), (max(loads), mean)
    return max(loads) / mean


# the workloads' causal shapes, plus one with a partial last head group
SHAPES = [(2, 16, 4096, 128), (4, 32, 2048, 128), (1, 16, 16384, 128), (4, 16, 4096, 128), (8, 12, 1000, 64),
          (3, 5, 777, 64)]


@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_forward_lists(B, H, N, d):
    BH = B * H
    cost = _fwd_units(BH, N)
    grid = min(len(cost), SMS)
    lists = fa.unit_lists(0, B, H, N, d, grid)
    ratio = _check(lists, cost, _fwd_position(BH, N, d), grid)
    if len(cost) >= 6 * grid:  # enough units per CTA: within 4% of the mean
        assert ratio <= 1.04, ratio


@pytest.mark.parametrize("B,H,N,d", [s for s in SHAPES if s[3] == 128])
def test_forward_lists_per_cta_pair(B, H, N, d):
    """The paired (two-SM) kernel's lists with the mask: the same units and
    builder, one worker per CTA pair (74 pairs on 148 SMs)."""
    BH = B * H
    cost = _fwd_units(BH, N)
    grid = min(len(cost), SMS // 2)
    lists = fa.unit_lists(0, B, H, N, d, grid)
    ratio = _check(lists, cost, _fwd_position(BH, N, d), grid)
    if len(cost) >= 6 * grid:
        assert ratio <= 1.04, ratio


@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_backward_lists(B, H, N, d):
    BH = B * H
    cost = _bwd_units(BH, N, d)
    grid = min(len(cost), SMS)
    lists = fa.unit_lists(1, B, H, N, d, grid)
    ratio = _check(lists, cost, {u: u for u in cost}, grid)
    if len(cost) >= 6 * grid:  # enough units per CTA: within 4% of the mean
        assert ratio <= 1.04, ratio


def test_single_unit_and_tiny_grids():
    assert fa.unit_lists(0, 1, 1, 256, 64, 1) == [[0]]
    assert fa.unit_lists(1, 1, 1, 256, 64, 2) is not None
    lists = fa.unit_lists(1, 1, 1, 256, 64, 2)
    assert sorted(u for L in lists for u in L) == [0, 1]


def test_more_units_than_the_lists_hold():
    # 1200 heads x 8 query-tile pairs (forward) and x 16 key tiles (backward)
    assert fa.unit_lists(0, 4, 300, 2048, 64, SMS) is None
    assert fa.unit_lists(1, 4, 300, 2048, 64, SMS) is None


def test_bad_arguments():
    lib = fa.load_library()
    import ctypes
    start = (ctypes.c_ushort * 200)()
    order = (ctypes.c_ushort * 4096)()
    s, o = ctypes.cast(start, ctypes.c_void_p), ctypes.cast(order, ctypes.c_void_p)
    assert lib.fa_unit_lists(2, 1, 1, 256, 64, 1, s, o, 4096) == EINVAL      # kind
    assert lib.fa_unit_lists(0, 1, 1, 256, 64, 0, s, o, 4096) == EINVAL      # grid
    assert lib.fa_unit_lists(0, 1, 1, 256, 64, 161, s, o, 4096) == EINVAL    # grid above the lists' CTAs
    assert lib.fa_unit_lists(0, 1, 1, 256, 32, 1, s, o, 4096) == EINVAL      # d
    assert lib.fa_unit_lists(0, 2, 16, 4096, 128, 148, s, o, 100) == EINVAL  # order too small
    assert lib.fa_unit_lists(0, 1, 1, 256, 64, 1, None, o, 4096) == EINVAL
