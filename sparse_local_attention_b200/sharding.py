"""Spreading one Sliding Tile Attention problem over several GPUs by heads.

Every (batch, head) slice of the attention is independent: a query attends
only to keys of its own slice, so no data crosses between slices ("Fast Video
Generation with Sliding Tile Attention", summary page, Methodology: each head
keeps its own window).  One problem therefore spreads over ranks by giving
each rank whole heads, with no exchange between them.

Heads with different windows cost different amounts: every query of head h
attends to keys_per_query(h) keys, so a head's forward (and backward) work is
proportional to that count.  partition_heads assigns heads in
longest-processing-time order -- the costliest head first, each to the rank
with the least work so far (ties to the lower rank) -- which gives every rank
one head of each window class when the classes divide evenly, as they do for
24 heads in three classes of 8 on 8 ranks.

This module only plans the split and selects tensor slices; it holds no
attention arithmetic.
"""
from __future__ import annotations

from typing import List, Sequence

import torch

from .workloads import Workload


def head_costs(wl: Workload) -> List[int]:
    """Keys per query of every head (its clamped window's tiles x tile volume)."""
    return [wl.keys_per_query(h) for h in range(wl.Hh)]


def partition_heads(costs: Sequence[int], world: int) -> List[List[int]]:
    """Heads of each rank (ascending), longest-processing-time order.

    Every head goes to exactly one rank.  With world > len(costs) some ranks
    get no head; callers that need work on every rank check for that."""
    if world < 1:
        raise ValueError("world must be >= 1")
    loads = [0] * world
    ranks: List[List[int]] = [[] for _ in range(world)]
    for h in sorted(range(len(costs)), key=lambda i: (-costs[i], i)):
        r = min(range(world), key=lambda i: (loads[i], i))
        ranks[r].append(h)
        loads[r] += costs[h]
    return [sorted(r) for r in ranks]


def shard_workload(wl: Workload, heads: Sequence[int]) -> Workload:
    """The sub-problem of the given heads: same latent, tiles and batch, those
    heads' windows, in the given order."""
    if not heads:
        raise ValueError("a shard needs at least one head")
    return wl.with_(name=f"{wl.name}/heads{list(heads)}", Hh=len(heads),
                    windows=tuple(tuple(wl.windows[h]) for h in heads))


def select_heads(x: torch.Tensor, heads: Sequence[int]) -> torch.Tensor:
    """The given heads of a [B, heads, ...] tensor, as a contiguous tensor."""
    return x[:, list(heads)].contiguous()
