"""Splitting one problem's heads over ranks (host logic, no GPU)."""
import os
import sys

import pytest
import torch

from sparse_local_attention_b200.sharding import head_costs, partition_heads, select_heads, shard_workload
from sparse_local_attention_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 5, 6, 7, 8, 16, 24])
def test_every_head_on_one_rank_and_loads_balanced(world):
    wl = WORKLOADS["dit720p_perhead"]
    costs = head_costs(wl)
    parts = partition_heads(costs, world)
    assert len(parts) == world
    assert sorted(h for p in parts for h in p) == list(range(wl.Hh))
    loads = [sum(costs[h] for h in p) for p in parts]
    # greedy longest-processing-time: no rank exceeds the mean by more than one head
    assert max(loads) <= sum(costs) / world + max(costs)
    # the sub-problems' work adds up to the whole problem's
    assert sum(shard_workload(wl, p).forward_flops() for p in parts) == wl.forward_flops()


def test_three_window_classes_on_eight_ranks():
    """24 heads in classes 1x3x3 / 3x3x5 / 5x5x5 (8 each): every rank gets one
    head of each class, so all ranks carry the same work."""
    wl = WORKLOADS["dit720p_perhead"]
    parts = partition_heads(head_costs(wl), 8)
    for p in parts:
        assert sorted(wl.windows[h] for h in p) == [(1, 3, 3), (3, 3, 5), (5, 5, 5)]
    assert len({shard_workload(wl, p).forward_flops() for p in parts}) == 1


def test_equal_heads_split_round_robin_and_excess_ranks_idle():
    assert partition_heads([5] * 6, 3) == [[0, 3], [1, 4], [2, 5]]
    assert partition_heads([1, 1], 3) == [[0], [1], []]
    assert partition_heads([], 2) == [[], []]
    with pytest.raises(ValueError):
        partition_heads([1], 0)


def test_shard_workload_and_slices():
    wl = WORKLOADS["tiny"].with_(Hh=4, windows=((1, 1, 1), (3, 3, 3), (2, 2, 2), (3, 1, 1)))
    sub = shard_workload(wl, [3, 1])
    assert sub.Hh == 2 and sub.windows == ((3, 1, 1), (3, 3, 3))
    assert (sub.T, sub.H, sub.W, sub.tile, sub.B, sub.d) == (wl.T, wl.H, wl.W, wl.tile, wl.B, wl.d)
    with pytest.raises(ValueError):
        shard_workload(wl, [])
    x = torch.arange(2 * 4 * 3 * 2, dtype=torch.float32).reshape(2, 4, 3, 2)
    y = select_heads(x, [3, 1])
    assert y.is_contiguous() and torch.equal(y[:, 0], x[:, 3]) and torch.equal(y[:, 1], x[:, 1])


def test_bench_refuses_more_ranks_than_heads():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(SystemExit):
        bench.rank_share(WORKLOADS["tiny"], 3, 0, "heads")  # 2 heads, 3 ranks
    wl, heads, job, scaling = bench.rank_share(WORKLOADS["tiny"], 1, 0, "heads")
    assert heads == [0, 1] and job == WORKLOADS["tiny"].forward_flops() and scaling == "strong"
    wl, heads, job, scaling = bench.rank_share(WORKLOADS["tiny"], 4, 2, "problem")
    assert heads is None and job == 4 * WORKLOADS["tiny"].forward_flops() and scaling == "weak"
