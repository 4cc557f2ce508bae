"""GPU backward parity: sta_backward (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs and outputs, fp32 accumulation, bf16 P and dS fed to
the tensor cores) on dQ, dK and dV: max-abs <= 2e-2, mean-abs <= 2e-3.

Besides the oracle comparisons, three identities of the gradients are checked
on every row at full size, where the oracle is too slow to visit every row:
    sum_j dV_j = sum_i dO_i           (rows of P sum to one)
    sum_j dK_j = 0                    (rows of dS sum to zero)
    dQ = 0 when all key rows are equal (same reason)
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload, make_inputs, tile_tokens, tiles_sample

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def geom_of(wl: Workload) -> Geometry:
    return Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))


def run_fwd_bwd(wl: Workload, q, k, v, do, tiled=False):
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True, tiled=tiled))
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = sta.sta_forward(plan, qd, kd, vd, check=True)
    dq, dk, dv = sta.sta_backward(plan, qd, kd, vd, o, lse, dod, check=True)
    torch.cuda.synchronize()
    return plan, (o, lse), (dq, dk, dv)


def compare(name, got, ref):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), name
    assert err.max() <= MAX_ABS, f"{name}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{name}: mean abs err {err.mean():.3e}"
    return err.max()


SMALL = {
    "tiny_workload": WORKLOADS["tiny"].with_(backward=True),
    "d128_tau64": Workload("a", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3)), backward=True),
    "d64_tau384_three_blocks": Workload("b", 2, 1, 64, 12, 16, 16, (6, 8, 8), ((3, 3, 3),), backward=True),
    "d128_permute_fallback": Workload("c", 1, 2, 128, 4, 12, 8, (2, 6, 4), ((3, 1, 2), (2, 2, 2)), backward=True),
    "d64_tau192_partial_block": Workload("d", 1, 2, 64, 6, 16, 24, (3, 8, 8), ((1, 1, 3), (2, 2, 2)), backward=True),
    # 2D (image) STA: one frame, 1 x 8 x 8 tiles
    "d64_image_2d": Workload("e", 1, 2, 64, 1, 32, 48, (1, 8, 8), ((1, 3, 3), (1, 5, 5)), backward=True),
    "d128_image_2d_tau256": Workload("f", 1, 1, 128, 1, 32, 64, (1, 16, 16), ((1, 1, 3),), backward=True),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_small_all_rows(name):
    wl = SMALL[name]
    q, k, v, do = make_inputs(wl, with_dout=True, seed=2)
    _, _, (dq, dk, dv) = run_fwd_bwd(wl, q, k, v, do)
    g = geom_of(wl)
    for bh in range(wl.B * wl.Hh):
        b, h = divmod(bh, wl.Hh)
        rdq, rdk, rdv = oracle.backward(g, q, k, v, do, bh)
        compare(f"dq[{bh}]", dq[b, h].double().cpu().numpy(), rdq)
        compare(f"dk[{bh}]", dk[b, h].double().cpu().numpy(), rdk)
        compare(f"dv[{bh}]", dv[b, h].double().cpu().numpy(), rdv)


def test_backward_tiled_layout_matches_raster():
    wl = SMALL["d128_tau64"]
    q, k, v, do = make_inputs(wl, with_dout=True, seed=4)
    plan, _, grads = run_fwd_bwd(wl, q, k, v, do)
    tq, tk, tv, tdo = (sta.sta_permute(plan, x.cuda()) for x in (q, k, v, do))
    plan_t = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True, tiled=True))
    o_t, lse_t = sta.sta_forward(plan_t, tq, tk, tv, check=True)
    g_t = sta.sta_backward(plan_t, tq, tk, tv, o_t, lse_t, tdo, check=True)
    for a, b in zip(grads, g_t):
        assert torch.equal(sta.sta_permute(plan, b, inverse=True), a)


def test_backward_is_deterministic():
    wl = SMALL["d64_tau384_three_blocks"]
    q, k, v, do = make_inputs(wl, with_dout=True, seed=5)
    _, _, g1 = run_fwd_bwd(wl, q, k, v, do)
    _, _, g2 = run_fwd_bwd(wl, q, k, v, do)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_finetune_sampled_rows():
    """The fine-tuning workload (2x16 heads, 16x64x64, tile 4x8x8, window
    3x5x5): dQ on 16 rows (first, last and 14 seeded) of each of 64 query
    tiles (8 corners + 56 seeded) for all 32 (batch, head) slices; dK/dV on 4
    rows of each of 64 key tiles for 4 seeded slices (each of those needs the
    oracle's LSE and D for almost every query of the slice)."""
    wl = WORKLOADS["finetune"]
    q, k, v, do = make_inputs(wl, with_dout=True)
    _, _, (dq, dk, dv) = run_fwd_bwd(wl, q, k, v, do)
    g = geom_of(wl)
    rng = np.random.default_rng(0)
    qtiles = tiles_sample(wl, 64, seed=0)
    assert len(qtiles) == 64
    dq_host = dq.cpu()
    for bh in range(wl.B * wl.Hh):
        rows = []
        for t in qtiles:
            toks = tile_tokens(wl, t)
            rows += [toks[0], toks[-1]] + list(rng.choice(toks[1:-1], 14, replace=False))
        rows = np.array(sorted(set(rows)))
        b, h = divmod(bh, wl.Hh)
        rdq, _, _ = oracle.backward(g, q, k, v, do, bh, q_rows=rows, k_rows=np.zeros(0, dtype=np.int64))
        compare(f"dq[{bh}]", dq_host[b, h, torch.as_tensor(rows)].double().numpy(), rdq)
    slices = [0, 17, 2 * wl.Hh - 1, 9]
    ktiles = tiles_sample(wl, 64, seed=1)
    for bh in slices:
        rows = []
        for t in ktiles:
            toks = tile_tokens(wl, t)
            rows += [toks[0], toks[-1]] + list(rng.choice(toks, 2, replace=False))
        rows = np.array(sorted(set(rows)))
        b, h = divmod(bh, wl.Hh)
        _, rdk, rdv = oracle.backward(g, q, k, v, do, bh, q_rows=np.zeros(0, dtype=np.int64), k_rows=rows)
        idx = torch.as_tensor(rows)
        compare(f"dk[{bh}]", dk[b, h, idx].double().cpu().numpy(), rdk)
        compare(f"dv[{bh}]", dv[b, h, idx].double().cpu().numpy(), rdv)


@pytest.mark.parametrize("name", ["finetune", "dit720p"])
def test_gradient_identities_full_scale(name):
    wl = WORKLOADS[name].with_(backward=True, B=1, Hh=4) if name == "dit720p" else WORKLOADS[name]
    q, k, v, do = make_inputs(wl, with_dout=True, seed=7)
    _, _, (dq, dk, dv) = run_fwd_bwd(wl, q, k, v, do)
    # sum over keys of dV equals the sum over queries of dO (per slice)
    sdv = dv.double().sum(2)
    sdo = do.cuda().double().sum(2)
    rel = (sdv - sdo).abs().max() / sdo.abs().max()
    assert rel < 5e-3, float(rel)
    # sum over keys of dK is zero (relative to the size of dK)
    sdk = dk.double().sum(2).abs().max() / dk.double().abs().sum(2).max()
    assert sdk < 5e-3, float(sdk)
    # equal key rows: dS rows sum to zero, so dQ vanishes
    k_eq = k[:, :, :1].expand_as(k).contiguous()
    _, _, (dq0, _, _) = run_fwd_bwd(wl, q, k_eq, v, do)
    assert dq0.float().abs().max() < 2e-3, float(dq0.float().abs().max())


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"].with_(backward=True), SMALL["d128_tau64"]], ids=lambda w: w.name)
def test_autograd_function_matches_the_abi_calls(wl):
    """sliding_tile_attention under autograd: its O equals sta_forward's and the
    gradients of sum(O * dO) equal sta_backward's for the same dO, bit for bit
    (the same deterministic kernels on the same inputs); without gradients it
    returns the same O."""
    q, k, v, do = (x.cuda() for x in make_inputs(wl, with_dout=True, seed=5))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    o_ref, lse_ref = sta.sta_forward(plan, q, k, v, check=True)
    g_ref = sta.sta_backward(plan, q, k, v, o_ref, lse_ref, do, check=True)
    qa, ka, va = (x.clone().requires_grad_() for x in (q, k, v))
    o = sta.sliding_tile_attention(qa, ka, va, wl.T, wl.H, wl.W, wl.tile, wl.windows)
    (o.float() * do.float()).sum().backward()
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o_ref)
    for name, got, ref in zip(("dq", "dk", "dv"), (qa.grad, ka.grad, va.grad), g_ref):
        assert torch.equal(got, ref), name
    with torch.no_grad():
        o_plain = sta.sliding_tile_attention(q, k, v, wl.T, wl.H, wl.W, wl.tile, wl.windows)
    torch.cuda.synchronize()
    assert torch.equal(o_plain, o_ref)
    plan.destroy()
