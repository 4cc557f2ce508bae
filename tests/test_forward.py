"""GPU forward parity: sta_forward (through the C ABI) against the fp64 oracle.

Tolerances (GPU bf16 inputs, fp32 accumulation, bf16 output) vs the fp64
oracle on the same bf16 inputs: max-abs <= 2e-2 and mean-abs <= 2e-3 on O.
LSE (fp32) within 2e-3 absolute.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload, make_inputs, tile_tokens, tiles_sample

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 2e-3


def geom_of(wl: Workload) -> Geometry:
    return Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))


def run_gpu(wl: Workload, q, k, v, tiled=False):
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False, tiled=tiled))
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = sta.sta_forward(plan, qd, kd, vd, check=True)
    torch.cuda.synchronize()
    return o, lse, plan


def compare_rows(wl, o_gpu, lse_gpu, q, k, v, rows):
    o_ref, lse_ref = oracle.forward(geom_of(wl), q, k, v, rows=rows)
    og = o_gpu.reshape(-1, wl.d)[torch.as_tensor(rows, device=o_gpu.device)].double().cpu().numpy()
    err = np.abs(og - o_ref)
    assert np.isfinite(og).all()
    assert err.max() <= MAX_ABS, f"max abs err {err.max()}"
    assert err.mean() <= MEAN_ABS, f"mean abs err {err.mean()}"
    if lse_gpu is not None:
        lg = lse_gpu.reshape(-1)[torch.as_tensor(rows, device=lse_gpu.device)].double().cpu().numpy()
        assert np.abs(lg - lse_ref).max() <= LSE_ABS, f"lse err {np.abs(lg - lse_ref).max()}"
    return err.max(), err.mean()


def sampled_rows(wl: Workload, n_tiles=64, rows_per_tile=None, bh_list=None, seed=0):
    tiles = tiles_sample(wl, n_tiles, seed)
    gen = np.random.default_rng(seed)
    rows = []
    bhs = range(wl.B * wl.Hh) if bh_list is None else bh_list
    for t in tiles:
        toks = tile_tokens(wl, t)
        if rows_per_tile is None or rows_per_tile >= len(toks):
            pick = toks
        else:
            extra = gen.choice(len(toks) - 2, size=rows_per_tile - 2, replace=False) + 1
            pick = [toks[0], toks[-1]] + [toks[i] for i in extra]
        for bh in bhs:
            rows.extend(bh * wl.N + n for n in pick)
    return np.array(sorted(rows), dtype=np.int64)


# ----------------------------------------------------------------- small cases
SMALL = {
    # name: (B, Hh, d, T, H, W, tile, windows)
    "tiny_workload": WORKLOADS["tiny"],
    "d128_tau64_two_pieces": Workload("a", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3))),
    "d64_tau192_partial_block": Workload("b", 2, 2, 64, 6, 16, 24, (3, 8, 8), ((1, 1, 3), (2, 2, 2))),
    "d128_tau48_boxes_of_16": Workload("c", 1, 3, 128, 6, 8, 12, (3, 4, 4), ((3, 3, 3), (1, 2, 3), (9, 9, 9))),
    "d64_tau384_three_blocks": Workload("d", 1, 2, 64, 12, 16, 16, (6, 8, 8), ((3, 3, 3), (1, 1, 1))),
    "d128_permute_fallback": Workload("e", 1, 2, 128, 4, 12, 8, (2, 6, 4), ((3, 1, 2), (2, 2, 2))),
    "d64_single_tile_grid": Workload("f", 2, 1, 64, 2, 8, 8, (2, 8, 8), ((3, 3, 3),)),
    "d128_tau8_tiny_tiles": Workload("g", 1, 2, 128, 4, 4, 8, (1, 2, 4), ((3, 3, 3), (2, 1, 2))),
    # 2D (image) STA: a one-frame latent with 1 x th x tw tiles
    "d64_image_2d": Workload("n", 1, 2, 64, 1, 32, 48, (1, 8, 8), ((1, 3, 3), (1, 5, 5))),
    "d128_image_2d_tau256": Workload("o", 1, 1, 128, 1, 64, 64, (1, 16, 16), ((1, 3, 3),)),
    # windows that are distinct for some tiles: their last blocks stay lone (split across warpgroups)
    "d128_lone_blocks_split": Workload("l", 1, 2, 128, 4, 8, 32, (2, 8, 8), ((1, 1, 2), (1, 1, 3))),
    "d64_lone_block_odd_chunks": Workload("m", 2, 1, 64, 2, 8, 40, (2, 8, 8), ((1, 1, 3),)),
    # tile volumes that are multiples of 128
    "d128_tau128_one_block": Workload("h", 1, 2, 128, 4, 16, 16, (2, 8, 8), ((3, 3, 3), (1, 2, 2))),
    "d128_tau256": Workload("i", 2, 1, 128, 8, 16, 24, (4, 8, 8), ((2, 3, 3),)),
    "d128_tau384_odd_blocks": Workload("j", 1, 2, 128, 12, 16, 16, (6, 8, 8), ((3, 3, 3), (1, 1, 1))),
    "d128_tau256_big_window": Workload("k", 1, 1, 128, 8, 24, 24, (4, 8, 8), ((5, 5, 5),)),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_all_rows(name):
    wl = SMALL[name]
    q, k, v = make_inputs(wl, seed=1)
    o, lse, _ = run_gpu(wl, q, k, v)
    rows = np.arange(wl.B * wl.Hh * wl.N)
    compare_rows(wl, o, lse, q, k, v, rows)


@pytest.mark.parametrize("name", ["d128_tau48_boxes_of_16", "d128_tau384_odd_blocks"])
def test_forward_tiled_layout_matches_raster(name):
    wl = SMALL[name]
    q, k, v = make_inputs(wl, seed=2)
    o, lse, plan = run_gpu(wl, q, k, v)
    qt, kt, vt = (sta.sta_permute(plan, x.cuda()) for x in (q, k, v))
    plan_t = sta.sta_plan_create(sta.Problem.from_workload(wl, tiled=True))
    o_t, lse_t = sta.sta_forward(plan_t, qt, kt, vt, check=True)
    o_back = sta.sta_permute(plan, o_t, inverse=True)
    torch.cuda.synchronize()
    assert torch.equal(o_back, o)


def test_forward_is_deterministic():
    wl = SMALL["d64_tau384_three_blocks"]
    q, k, v = make_inputs(wl, seed=3)
    o1, l1, _ = run_gpu(wl, q, k, v)
    o2, l2, _ = run_gpu(wl, q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ----------------------------------------------------------------- closed forms at full scale
@pytest.mark.parametrize("name", ["dit720p", "dit720p_perhead", "finetune"])
def test_one_hot_tile_coordinates_full_scale(name):
    """Q = 0 and V = one-hot tile coordinates: every output channel is exactly
    1/w' inside the window (per dimension) and 0 outside.  Checks every row of
    every head: a missing or extra key tile anywhere shows up here."""
    wl = WORKLOADS[name]
    gt, gh, gw = wl.grid
    tt, th, tw = wl.tile
    n = torch.arange(wl.N)
    t, h, w = n // (wl.H * wl.W), (n // wl.W) % wl.H, n % wl.W
    v1 = torch.zeros(wl.N, wl.d)
    v1[n, t // tt] = 1
    v1[n, gt + h // th] = 1
    v1[n, gt + gh + w // tw] = 1
    v = v1.to(torch.bfloat16).expand(wl.B, wl.Hh, wl.N, wl.d).contiguous().cuda()
    q = torch.zeros_like(v)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    o, lse = sta.sta_forward(plan, q, v, v, check=True)
    torch.cuda.synchronize()
    G = (gt, gh, gw)
    qtile = torch.stack([t // tt, h // th, w // tw], 1)
    for head in range(wl.Hh):
        win = wl.windows[head]
        expect = torch.zeros(wl.N, wl.d)
        base = 0
        for dim in range(3):
            wl_d = min(win[dim], G[dim])
            s = (qtile[:, dim] - wl_d // 2).clamp(min=0).clamp(max=G[dim] - wl_d)
            for x in range(G[dim]):
                inside = (s <= x) & (x < s + wl_d)
                expect[:, base + x] = inside.float() / wl_d
            base += G[dim]
        got = o[:, head].float().cpu()
        err = (got - expect).abs()
        assert err.max() <= 4e-3, (head, err.max())
        assert torch.allclose(lse[:, head].cpu(), torch.full_like(lse[:, head].cpu(), math.log(wl.keys_per_query(head))),
                              atol=1e-3)


# ----------------------------------------------------------------- sampled oracle on the large workloads
# Whole query tiles: the 8 corner tiles of the grid (where the window is
# shifted inward) and 56 seeded others, every row of each.  Heads: every head
# of the 720p and fine-tuning workloads; on the per-head workload two heads of
# each window class (1x3x3, 3x3x5, 5x5x5).  The full-window workload (115200
# keys per row) is compared with the library's dense attention on every row
# and with the oracle on sampled rows of the same tiles.
LARGE = {
    # name: (rows per tile or None for all, heads or None for all)
    "dit720p": (None, None),
    "dit720p_perhead": (None, (0, 7, 8, 15, 16, 23)),
    "finetune": (None, None),
    "dit720p_full": (2, None),
}


@pytest.mark.parametrize("name", list(LARGE))
def test_forward_large_sampled(name):
    wl = WORKLOADS[name]
    rows_per_tile, heads = LARGE[name]
    q, k, v = make_inputs(wl)
    o, lse, _ = run_gpu(wl, q, k, v)
    bh_list = None if heads is None else [b * wl.Hh + h for b in range(wl.B) for h in heads]
    rows = sampled_rows(wl, 64, rows_per_tile, bh_list=bh_list)
    if rows_per_tile is None:
        assert len(rows) == 64 * wl.tile_volume * (wl.B * wl.Hh if heads is None else len(bh_list))
    compare_rows(wl, o, lse, q, k, v, rows)
    if name == "dit720p_full":
        # the whole output against the library's dense attention on the GPU
        ref = torch.nn.functional.scaled_dot_product_attention(q.cuda(), k.cuda(), v.cuda())
        err = (o.float() - ref.float()).abs()
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


def test_tiny_workload_full_oracle():
    wl = WORKLOADS["tiny"]
    q, k, v = make_inputs(wl)
    o, lse, _ = run_gpu(wl, q, k, v)
    compare_rows(wl, o, lse, q, k, v, np.arange(wl.B * wl.Hh * wl.N))


# ----------------------------------------------------------------- host tensors (sta_forward_host)
@pytest.mark.parametrize("name,pinned", [
    ("d128_tau384_odd_blocks", True),     # 2 slices, pairs and lone blocks
    ("d64_tau192_partial_block", True),   # batch 2: 4 slices in 4 groups
    ("d128_permute_fallback", True),      # gather path: copied whole, not pipelined
    ("d128_tau256", True),                # two query blocks per tile
    ("tiny_workload", False),             # pageable host memory
])
def test_forward_host_equals_device_call(name, pinned):
    wl = SMALL[name]
    q, k, v = make_inputs(wl, seed=4)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    _host_vs_device(plan, q, k, v, pinned)


def test_forward_host_tile_major_tensors():
    """sta_forward_host on a plan for tile-major tensors (the slice groups
    are contiguous in either token order)."""
    wl = SMALL["d64_tau384_three_blocks"]
    q, k, v = make_inputs(wl, seed=8)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False, tiled=True))
    _host_vs_device(plan, q, k, v, True)


def _host_vs_device(plan, q, k, v, pinned):
    o_dev, lse_dev = sta.sta_forward(plan, q.cuda(), k.cuda(), v.cuda(), check=True)
    qh, kh, vh = (x.pin_memory() if pinned else x for x in (q, k, v))
    o_h, lse_h = sta.sta_forward_host(plan, qh, kh, vh, check=True)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(lse_h, lse_dev.cpu())


def test_forward_host_full_scale_groups():
    """32 slices in 24 groups of one or two (fine-tuning shapes): the pipelined host call
    returns exactly the device call's outputs."""
    wl = WORKLOADS["finetune"]
    q, k, v = make_inputs(wl, seed=6)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    o_dev, lse_dev = sta.sta_forward(plan, q.cuda(), k.cuda(), v.cuda(), check=True)
    o_h, lse_h = sta.sta_forward_host(plan, q.pin_memory(), k.pin_memory(), v.pin_memory(), check=True)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(lse_h, lse_dev.cpu())
