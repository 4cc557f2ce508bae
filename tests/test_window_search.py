"""Per-head window search: the selection rule on the host (fake forward), and
the search through sta_forward on the GPU against the fp64 oracle."""
import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.window_search import clamped_keys, relative_errors, search_windows
from sparse_local_attention_b200.workloads import Workload, positional_field


def test_selection_rule_with_fake_forward():
    """Every head takes the cheapest candidate within budget; candidates are
    tried by clamped key count, not in the given order; a head no candidate
    satisfies gets the whole grid."""
    B, heads, T, H, W, d = 1, 3, 4, 16, 16, 8
    tile, N = (2, 4, 4), 4 * 16 * 16
    ref = torch.ones(B, heads, N, d, dtype=torch.float64)
    table = {  # relative error per head of each window's output
        (1, 1, 1): [0.30, 0.01, 0.50],
        (2, 3, 3): [0.04, 0.001, 0.20],
        (2, 4, 4): [0.0, 0.0, 0.0],   # the whole 2x4x4 grid
        (1, 3, 3): [0.06, 0.002, 0.30],
    }
    calls = []

    def fake_forward(window):
        calls.append(window)
        e = torch.tensor(table[window], dtype=torch.float64).view(1, heads, 1, 1)
        return ref * (1 + e)

    cands = [(2, 3, 3), (1, 1, 1), (1, 3, 3)]  # not sorted by cost
    res = search_windows(ref, ref, ref, T, H, W, tile, cands, budget=0.05, reference=ref, forward=fake_forward)
    assert calls == [(1, 1, 1), (1, 3, 3), (2, 3, 3), (2, 4, 4)]
    assert res.windows == [(2, 3, 3), (1, 1, 1), (2, 4, 4)]
    assert res.errors == pytest.approx([0.04, 0.01, 0.0])
    assert res.keys_per_query == [2 * 3 * 3 * 32, 32, 2 * 4 * 4 * 32]


def test_search_stops_once_every_head_is_decided():
    ref = torch.ones(1, 2, 64, 4, dtype=torch.float64)
    calls = []

    def fake_forward(window):
        calls.append(window)
        return ref

    res = search_windows(ref, ref, ref, 1, 8, 8, (1, 4, 4), [(1, 1, 1), (1, 2, 2)], budget=0.0, reference=ref,
                         forward=fake_forward)
    assert calls == [(1, 1, 1)] and res.windows == [(1, 1, 1), (1, 1, 1)]


def test_clamped_keys_and_relative_errors():
    assert clamped_keys((9, 3, 1), (2, 4, 4), (3, 4, 4)) == 3 * 3 * 1 * 32
    a = torch.zeros(2, 2, 3, 4)
    b = torch.ones(2, 2, 3, 4)
    b[:, 1] *= 2
    assert relative_errors(b, b) == [0.0, 0.0]
    assert relative_errors(a, b) == pytest.approx([1.0, 1.0])


@pytest.mark.gpu
def test_search_on_gpu_meets_budget_and_is_minimal():
    """The search through sta_forward on a 1024-token latent, against the
    fp64 oracle: the reference is the oracle's whole-grid output (full
    attention, itself checked against the library's dense attention), and the
    chosen per-head windows, run together in one plan, match the oracle's
    output for those windows element by element."""
    import numpy as np

    import oracle
    # Attention that is local to a different extent in each head: queries and
    # keys share the smooth positional field F (so q.k peaks where the two
    # tokens are close), the query scaled by 0.5, 2 and 8 in the three heads,
    # plus a little noise; values are N(0, 1).  (Seed 5, drawn in the order
    # q noise, k noise, v.)
    wl = Workload("ws", 1, 3, 64, 4, 16, 16, (2, 4, 4), ((1, 1, 1),) * 3, field_amplitude=1.0)
    F = positional_field(wl)
    gen = torch.Generator().manual_seed(5)
    alphas = (0.5, 2.0, 8.0)
    q = torch.stack([a * F + 0.1 * torch.randn(F.shape, generator=gen) for a in alphas])[None].to(torch.bfloat16)
    k = torch.stack([F + 0.1 * torch.randn(F.shape, generator=gen) for _ in alphas])[None].to(torch.bfloat16)
    v = torch.randn(1, 3, wl.N, wl.d, generator=gen).to(torch.bfloat16)
    full = wl.with_(windows=(wl.grid,) * wl.Hh)
    geom = lambda w: oracle.Geometry(w.B, w.Hh, w.d, w.T, w.H, w.W, tuple(w.tile), tuple(w.windows))
    ref64, _ = oracle.forward(geom(full), q, k, v)
    ref = torch.from_numpy(ref64).view(q.shape).cuda()
    q, k, v = (x.cuda() for x in (q, k, v))
    sdpa = torch.nn.functional.scaled_dot_product_attention(q, k, v).double()
    assert (sdpa - ref).abs().max().item() <= 2e-2 and (sdpa - ref).abs().mean().item() <= 2e-3
    cands = [(1, 1, 1), (1, 3, 3), (2, 3, 3), (2, 4, 4)]
    # with these inputs the oracle's relative errors put the three heads'
    # cheapest windows at 2x4x4 (the whole grid), 2x3x3 and 1x1x1, each
    # candidate at least 0.04 away from the budget
    budget = 0.28
    res = search_windows(q, k, v, wl.T, wl.H, wl.W, wl.tile, cands, budget, reference=ref)
    assert len(set(res.windows)) == 3, res.windows  # the heads take different windows
    # the chosen per-head windows, run together in one plan, stay within budget
    plan = sta.sta_plan_create(sta.Problem(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, wl.tile, res.windows))
    o, lse = sta.sta_forward(plan, q, k, v, check=True)
    errs = relative_errors(o, ref)
    assert all(e <= budget for e in errs), errs
    # a head's output does not depend on the other heads' windows
    assert errs == pytest.approx(res.errors, rel=0, abs=1e-12)
    # ... and it is the oracle's output for those windows, element by element
    o_or, lse_or = oracle.forward(geom(wl.with_(windows=tuple(res.windows))), q, k, v)
    e = np.abs(o.reshape(-1, wl.d).double().cpu().numpy() - o_or)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
    assert np.abs(lse.reshape(-1).double().cpu().numpy() - lse_or).max() <= 2e-3
    # and every cheaper candidate that was tried misses the budget for that head
    for h, w in enumerate(res.windows):
        for cand, e in res.tried:
            if clamped_keys(cand, wl.tile, wl.grid) < clamped_keys(w, wl.tile, wl.grid):
                assert e[h] > budget, (h, cand, e[h])
