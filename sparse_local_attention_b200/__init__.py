"""Sliding Tile Attention for NVIDIA B200 (sm_100a).

The compute path lives in libsta.so (C ABI: include/sta.h); ``sta`` is its thin
ctypes binding.  ``workloads`` holds the seeded synthetic problem shapes.
"""
from .sta import (Plan, Problem, StaError, sliding_tile_attention, sta_backward, sta_forward, sta_forward_host,
                  sta_permute,
                  sta_plan_create, sta_plan_destroy, sta_plan_kv_tiles, sta_plan_q_tiles,
                  sta_plan_workspace_size, sta_set_wait_limit_ns)

__all__ = ["Plan", "Problem", "StaError", "sliding_tile_attention", "sta_backward", "sta_forward", "sta_forward_host",
           "sta_permute",
           "sta_plan_create", "sta_plan_destroy", "sta_plan_kv_tiles", "sta_plan_q_tiles",
           "sta_plan_workspace_size", "sta_set_wait_limit_ns"]
