"""The planner's work lists (host logic, no GPU): what the persistent kernels
walk.  Every query block and every key block is covered exactly once, block
pairs share their key tiles, lone blocks come last, and each list is in the
cost order the launches assume."""
import math

import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload

CASES = {
    "tiny": WORKLOADS["tiny"],
    "dit720p": WORKLOADS["dit720p"],
    "dit720p_perhead": WORKLOADS["dit720p_perhead"],
    "finetune": WORKLOADS["finetune"],
    "tau192_two_blocks_ragged": Workload("a", 2, 3, 64, 6, 16, 24, (3, 8, 8), ((1, 1, 3), (2, 2, 2), (3, 1, 1))),
    "tau64_one_block": Workload("b", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3))),
    "image_2d": Workload("c", 1, 2, 64, 1, 32, 48, (1, 8, 8), ((1, 3, 3), (1, 5, 5))),
    "many_slices": Workload("d", 3, 5, 64, 4, 8, 8, (4, 8, 8), ((1, 1, 1),) * 5),
}


def _plan(wl):
    return sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True, host_only=True))


def _lists(plan, wl):
    """Per head: [n_tiles][per_tile] KV-tile lists as tuples."""
    out = []
    for h in range(wl.Hh):
        kv = sta.sta_plan_kv_tiles(plan, h)
        out.append([tuple(r) for r in kv.tolist()])
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_forward_items(name):
    wl = CASES[name]
    plan = _plan(wl)
    nb = math.ceil(wl.tile_volume / 128)
    items, n_lone = sta.sta_plan_work_items(plan, sta.STA_WORK_FORWARD)
    items = items.tolist()
    lists = _lists(plan, wl)
    seen = {}
    for s, a, b, zero in items:
        assert zero == 0
        for blk in (a, b):
            if blk >= 0:
                key = (s, blk)
                assert key not in seen, f"block {key} twice"
                seen[key] = True
        if b >= 0:
            h = s % wl.Hh
            assert lists[h][a // nb] == lists[h][b // nb], "paired blocks attend to different key tiles"
            same_tile = a // nb == b // nb
            assert (same_tile and a % nb % 2 == 0 and b == a + 1) or \
                   (not same_tile and a % nb == nb - 1 and b % nb == nb - 1), (a, b)
    assert len(seen) == wl.B * wl.Hh * wl.n_tiles * nb, "some query block is missing"
    # lone blocks (B = -1) are exactly the last n_lone items
    lone_flags = [b < 0 for _, _, b, _ in items]
    assert lone_flags == [False] * (len(items) - n_lone) + [True] * n_lone
    # each part in non-increasing cost (blocks x key tiles)
    count = [len(lists[h][0]) for h in range(wl.Hh)]
    cost = [(2 if b >= 0 else 1) * count[s % wl.Hh] for s, _, b, _ in items]
    pairs, lone = cost[: len(items) - n_lone], cost[len(items) - n_lone:]
    assert pairs == sorted(pairs, reverse=True) and lone == sorted(lone, reverse=True)


def test_lone_blocks_of_the_720p_workload():
    """Tiles of 384 tokens have three blocks; the third pairs across tiles whose
    clamped windows coincide.  On the 5 x 6 x 10 grid with 3 x 3 x 3 windows,
    12 tiles per head have no such partner."""
    wl = WORKLOADS["dit720p"]
    _, n_lone = sta.sta_plan_work_items(_plan(wl), sta.STA_WORK_FORWARD)
    assert n_lone == 12 * wl.Hh


@pytest.mark.parametrize("name", list(CASES))
def test_host_items_are_the_forward_items_by_slice_group(name):
    wl = CASES[name]
    plan = _plan(wl)
    items, _ = sta.sta_plan_work_items(plan, sta.STA_WORK_FORWARD)
    host, _ = sta.sta_plan_work_items(plan, sta.STA_WORK_FORWARD_HOST)
    assert sorted(map(tuple, items.tolist())) == sorted(map(tuple, host.tolist()))
    slices = wl.B * wl.Hh
    groups = min(slices, 24)
    group_of = {}
    for g in range(groups):
        for s in range(slices * g // groups, slices * (g + 1) // groups):
            group_of[s] = g
    seq = [group_of[s] for s, _, _, _ in host.tolist()]
    assert seq == sorted(seq), "slice groups interleave"
    for g in range(groups):
        lone = [b < 0 for s, _, b, _ in host.tolist() if group_of[s] == g]
        assert lone == sorted(lone), "a group's lone blocks must follow its pairs"


@pytest.mark.parametrize("name", list(CASES))
def test_backward_items(name):
    wl = CASES[name]
    plan = _plan(wl)
    nb = math.ceil(wl.tile_volume / 128)
    every = sorted((s, blk) for s in range(wl.B * wl.Hh) for blk in range(wl.n_tiles * nb))
    kv, _ = sta.sta_plan_work_items(plan, sta.STA_WORK_DKDV)
    dq, _ = sta.sta_plan_work_items(plan, sta.STA_WORK_DQ)
    assert sorted(map(tuple, kv.tolist())) == every
    assert sorted(map(tuple, dq.tolist())) == every
    # dK/dV items: slice by slice, within a slice longest inverse list first
    inv = [sta.sta_plan_q_tiles(plan, h)[0] for h in range(wl.Hh)]
    keyed = [(s, -int(inv[s % wl.Hh][blk // nb + 1] - inv[s % wl.Hh][blk // nb])) for s, blk in kv.tolist()]
    assert keyed == sorted(keyed)
    # dQ items: costliest heads first
    count = [len(sta.sta_plan_kv_tiles(plan, h)[0]) for h in range(wl.Hh)]
    costs = [count[s % wl.Hh] for s, _ in dq.tolist()]
    assert costs == sorted(costs, reverse=True)


def test_forward_only_plan_has_no_backward_items_and_bad_kind_is_refused():
    wl = CASES["tiny"]
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False, host_only=True))
    assert sta.sta_plan_work_items(plan, sta.STA_WORK_DKDV)[0].shape == (0, 2)
    with pytest.raises(sta.StaError):
        sta.sta_plan_work_items(plan, 7)
