"""Planner checks on the host (no GPU): the KV-tile lists and inverse lists the
library builds must be bit-exact against the oracle's per-token membership."""
import numpy as np
import pytest

import oracle
from oracle import Geometry
from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS

CASES = [
    # (T, H, W, tile, windows)
    (6, 16, 16, (2, 4, 4), [(3, 3, 3), (1, 1, 1)]),
    (4, 6, 8, (2, 2, 2), [(1, 3, 2), (2, 2, 4), (5, 5, 5)]),
    (3, 8, 8, (1, 4, 2), [(7, 7, 7), (2, 3, 1)]),
    (5, 4, 12, (1, 2, 4), [(2, 1, 2), (4, 2, 1)]),
]


def host_plan(T, H, W, tile, windows, backward=True, d=64):
    return sta.sta_plan_create(sta.Problem(1, len(windows), d, T, H, W, tile, windows, backward=backward,
                                           host_only=True))


def oracle_tile_sets(T, H, W, tile, windows, head):
    """Key tiles the oracle's membership marks for the first token of each
    query tile (every token of a tile has the same window)."""
    g = Geometry(1, len(windows), 8, T, H, W, tile, tuple(windows))
    m = oracle.mask(g, head)
    gt, gh, gw = T // tile[0], H // tile[1], W // tile[2]
    n = np.arange(T * H * W)
    t, h, w = n // (H * W), (n // W) % H, n % W
    tile_of = (t // tile[0] * gh + h // tile[1]) * gw + w // tile[2]
    out = []
    for q in range(gt * gh * gw):
        tok = np.nonzero(tile_of == q)[0]
        rows = m[tok]
        assert (rows == rows[0]).all(), "window differs inside a tile"
        out.append(sorted(set(tile_of[rows[0]].tolist())))
    return out


@pytest.mark.parametrize("case", CASES)
def test_kv_lists_bit_exact_against_oracle_membership(case):
    T, H, W, tile, windows = case
    plan = host_plan(T, H, W, tile, windows)
    for head in range(len(windows)):
        lists = sta.sta_plan_kv_tiles(plan, head).numpy()
        ref = oracle_tile_sets(T, H, W, tile, windows, head)
        assert lists.shape == (len(ref), len(ref[0]))
        for q, r in enumerate(ref):
            assert lists[q].tolist() == r


@pytest.mark.parametrize("case", CASES)
def test_inverse_lists_are_the_transpose(case):
    T, H, W, tile, windows = case
    plan = host_plan(T, H, W, tile, windows)
    for head in range(len(windows)):
        lists = sta.sta_plan_kv_tiles(plan, head).numpy()
        off, idx = sta.sta_plan_q_tiles(plan, head)
        off, idx = off.numpy(), idx.numpy()
        n_tiles = lists.shape[0]
        assert off[-1] == lists.size  # every (q, k) pair appears once
        for k in range(n_tiles):
            qs = idx[off[k]:off[k + 1]].tolist()
            assert qs == sorted(q for q in range(n_tiles) if k in lists[q])


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_list_sizes(name):
    wl = WORKLOADS[name]
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True, host_only=True))
    assert plan.n_tiles == wl.n_tiles and plan.tile_volume == wl.tile_volume
    for head in sorted({0, wl.Hh - 1, wl.Hh // 2}):
        lists = sta.sta_plan_kv_tiles(plan, head)
        assert lists.shape[1] * wl.tile_volume == wl.keys_per_query(head)
        assert (lists >= 0).all() and (lists < wl.n_tiles).all()
        off, idx = sta.sta_plan_q_tiles(plan, head)
        assert int(off[-1]) == wl.n_tiles * lists.shape[1]


def test_dit720p_window_starts():
    """Along T (5 tiles, w=3) the windows start at 0,0,1,2,2; along W (10
    tiles) at 0,0,1,...,7,7 -- the border shift keeps every window full."""
    wl = WORKLOADS["dit720p"]
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, host_only=True))
    lists = sta.sta_plan_kv_tiles(plan, 0).numpy()
    gt, gh, gw = wl.grid
    starts_t = [lists[(qt * gh) * gw][0] // (gh * gw) for qt in range(gt)]
    starts_w = [lists[qw][0] % gw for qw in range(gw)]
    assert starts_t == [0, 0, 1, 2, 2]
    assert starts_w == [0, 0, 1, 2, 3, 4, 5, 6, 7, 7]
