"""Pins for the fp64 CPU oracle (no GPU).

The oracle follows the definition of Sliding Tile Attention ("Fast Video
Generation with Sliding Tile Attention", Abstract; summary page, Methodology
and Novelty).  None of the pages prints a worked example, so each check below
ties the oracle to something other than itself:

* an N x N mask built from a different statement of the window rule (the
  valid window whose centre is nearest the query tile, ties to the lower
  start) + torch's fp64 scaled_dot_product_attention on that mask;
* full 3D attention when the window covers the whole tile grid;
* probabilities of a row summing to one;
* a 1x1x1 window reducing to attention inside each tile;
* invariance / equivariance under permutations of tokens within tiles;
* closed forms: constant values, zero queries (uniform weights), and one-hot
  tile coordinates that reveal the window's extent along each dimension;
* torch autograd of the masked attention, and central finite differences,
  for the backward.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import Geometry


def geom(T, H, W, tile, windows, B=1, d=16):
    return Geometry(B=B, Hh=len(windows), d=d, T=T, H=H, W=W, tile=tuple(tile),
                    windows=tuple(tuple(w) for w in windows))


def rand_inputs(g: Geometry, seed=0, with_dout=False):
    gen = torch.Generator().manual_seed(seed)
    shape = (g.B, g.Hh, g.N, g.d)
    out = [torch.randn(shape, generator=gen).to(torch.bfloat16) for _ in range(4 if with_dout else 3)]
    return out


# ---------------------------------------------------------------------------
# Independent statement of the window: nearest-centre valid window.
# ---------------------------------------------------------------------------
def nearest_start(qtile: int, w: int, G: int) -> int:
    """Among all starts s with the window [s, s+w) inside [0, G), the one whose
    centre s + (w-1)/2 is nearest qtile; ties go to the smaller s."""
    w = min(w, G)
    best, best_dist = None, None
    for s in range(0, G - w + 1):
        dist = abs(s + (w - 1) / 2.0 - qtile)
        if best is None or dist < best_dist - 1e-12:
            best, best_dist = s, dist
    return best


def brute_mask(g: Geometry, head: int) -> np.ndarray:
    tt, th, tw = g.tile
    G = (g.T // tt, g.H // th, g.W // tw)
    coords = np.array([(t, h, w) for t in range(g.T) for h in range(g.H) for w in range(g.W)])
    tiles = coords // np.array([tt, th, tw])
    win = g.windows[head]
    m = np.ones((g.N, g.N), dtype=bool)
    for dim in range(3):
        wl = min(win[dim], G[dim])
        starts = np.array([nearest_start(int(q), win[dim], G[dim]) for q in range(G[dim])])
        s = starts[tiles[:, dim]][:, None]
        kt = tiles[:, dim][None, :]
        m &= (kt >= s) & (kt < s + wl)
    return m


def torch_masked(g: Geometry, q, k, v, masks, scale=None):
    """Dense fp64 attention with boolean masks per head, via the library SDPA."""
    scale = 1.0 / math.sqrt(g.d) if scale is None else scale
    qd, kd, vd = (x.double() for x in (q, k, v))
    mask = torch.stack([torch.from_numpy(m) for m in masks])[None]  # [1, Hh, N, N]
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale)
    s = torch.einsum("bhnd,bhmd->bhnm", qd, kd) * scale
    lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
    return o, lse


SMALL_CASES = [
    # (T, H, W, tile, windows)  -- odd, even, oversized and 1-tile windows
    (6, 16, 16, (2, 4, 4), [(3, 3, 3), (3, 3, 3)]),          # the tiny workload (3x4x4 grid)
    (2, 2, 2, (2, 2, 2), [(1, 1, 1), (3, 3, 3)]),            # 1x1x1 grid
    (4, 6, 8, (2, 2, 2), [(1, 3, 2), (2, 2, 4), (5, 5, 5)]),  # 2x3x4 grid
    (3, 8, 8, (1, 2, 2), [(7, 7, 7), (2, 3, 1), (1, 1, 1)]),  # 3x4x4 grid
    (5, 4, 6, (1, 2, 3), [(2, 1, 2), (4, 2, 1)]),            # 5x2x2 grid, even widths
    (1, 8, 12, (1, 2, 2), [(1, 3, 3), (1, 2, 5)]),           # 2D (image): one frame, 1x4x6 grid
]


@pytest.mark.parametrize("case", SMALL_CASES)
def test_mask_matches_nearest_centre_rule(case):
    T, H, W, tile, windows = case
    g = geom(T, H, W, tile, windows)
    for h in range(g.Hh):
        assert np.array_equal(oracle.mask(g, h), brute_mask(g, h))


@pytest.mark.parametrize("case", SMALL_CASES)
def test_forward_matches_masked_sdpa(case):
    T, H, W, tile, windows = case
    g = geom(T, H, W, tile, windows, B=2)
    q, k, v = rand_inputs(g, seed=3)
    o, lse = oracle.forward(g, q, k, v)
    ref_o, ref_lse = torch_masked(g, q, k, v, [brute_mask(g, h) for h in range(g.Hh)])
    np.testing.assert_allclose(o, ref_o.reshape(-1, g.d).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.reshape(-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", SMALL_CASES[:3])
def test_exhaustive_and_box_enumeration_agree_bitwise(case):
    T, H, W, tile, windows = case
    g = geom(T, H, W, tile, windows)
    q, k, v = rand_inputs(g, seed=5)
    o1, l1 = oracle.forward(g, q, k, v, exhaustive=True)
    o2, l2 = oracle.forward(g, q, k, v, exhaustive=False)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_full_window_equals_full_attention():
    g = geom(6, 8, 8, (2, 4, 4), [(3, 2, 2), (9, 9, 9)])  # grid 3x2x2: both windows cover it
    q, k, v = rand_inputs(g, seed=7)
    o, lse = oracle.forward(g, q, k, v)
    qd, kd, vd = (x.double() for x in (q, k, v))
    ref = F.scaled_dot_product_attention(qd, kd, vd)  # no mask at all
    np.testing.assert_allclose(o, ref.reshape(-1, g.d).numpy(), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(torch.einsum("bhnd,bhmd->bhnm", qd, kd) / math.sqrt(g.d), -1)
    np.testing.assert_allclose(lse, ref_lse.reshape(-1).numpy(), rtol=0, atol=1e-12)


def test_probabilities_sum_to_one_and_vanish_outside():
    g = geom(4, 6, 8, (2, 2, 2), [(1, 3, 2), (5, 5, 5)])
    q, k, v = rand_inputs(g, seed=11)
    for row in [0, 17, g.N - 1, g.N + 5, 2 * g.N - 1]:
        p = oracle.probs(g, q, k, v, row)
        head = row // g.N
        m = brute_mask(g, head)[row % g.N]
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p[~m] == 0.0) and np.all(p[m] > 0.0)


def test_single_tile_window_is_per_tile_attention():
    g = geom(4, 8, 8, (2, 4, 4), [(1, 1, 1)], B=1, d=32)
    q, k, v = rand_inputs(g, seed=13)
    o, _ = oracle.forward(g, q, k, v)
    qd, kd, vd = (x.double()[0, 0] for x in (q, k, v))
    ref = torch.zeros(g.N, g.d, dtype=torch.float64)
    tt, th, tw = g.tile
    for a, b, c in itertools.product(range(g.T // tt), range(g.H // th), range(g.W // tw)):
        idx = torch.tensor([(t * g.H + h) * g.W + w
                            for t in range(a * tt, a * tt + tt)
                            for h in range(b * th, b * th + th)
                            for w in range(c * tw, c * tw + tw)])
        ref[idx] = F.scaled_dot_product_attention(qd[idx][None], kd[idx][None], vd[idx][None])[0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def _within_tile_perm(g: Geometry, seed: int) -> torch.Tensor:
    """A permutation of token indices that moves tokens only within their tile."""
    gen = torch.Generator().manual_seed(seed)
    tt, th, tw = g.tile
    perm = torch.arange(g.N)
    for a, b, c in itertools.product(range(g.T // tt), range(g.H // th), range(g.W // tw)):
        idx = torch.tensor([(t * g.H + h) * g.W + w
                            for t in range(a * tt, a * tt + tt)
                            for h in range(b * th, b * th + th)
                            for w in range(c * tw, c * tw + tw)])
        perm[idx] = idx[torch.randperm(len(idx), generator=gen)]
    return perm


def test_within_tile_permutation_invariance():
    g = geom(6, 8, 8, (2, 4, 4), [(1, 2, 1), (3, 3, 3)])
    q, k, v = rand_inputs(g, seed=17)
    perm = _within_tile_perm(g, 1)
    o, lse = oracle.forward(g, q, k, v)
    # keys and values permuted together inside tiles: output unchanged
    o2, lse2 = oracle.forward(g, q, k[:, :, perm], v[:, :, perm])
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    # queries, keys and values permuted together: output permuted the same way
    o3, _ = oracle.forward(g, q[:, :, perm], k[:, :, perm], v[:, :, perm])
    o3 = o3.reshape(g.B, g.Hh, g.N, g.d)
    o = o.reshape(g.B, g.Hh, g.N, g.d)
    np.testing.assert_allclose(o3, o[:, :, perm.numpy()], rtol=0, atol=1e-12)


def test_constant_value_rows_closed_form():
    g = geom(4, 8, 8, (2, 4, 4), [(1, 3, 1), (2, 2, 2)])
    q, k, _ = rand_inputs(g, seed=19)
    row = torch.linspace(-2, 2, g.d).to(torch.bfloat16)
    v = row.expand(g.B, g.Hh, g.N, g.d).contiguous()
    o, _ = oracle.forward(g, q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(row.double().numpy(), o.shape), rtol=0, atol=1e-13)


def test_zero_query_gives_window_mean_and_log_count():
    g = geom(6, 8, 12, (2, 2, 3), [(3, 3, 3), (1, 2, 4)])
    _, k, v = rand_inputs(g, seed=23)
    q = torch.zeros_like(k)
    o, lse = oracle.forward(g, q, k, v)
    vd = v.double().numpy()
    for h in range(g.Hh):
        m = brute_mask(g, h)
        mean = (m.astype(np.float64) @ vd[0, h]) / m.sum(1, keepdims=True)
        np.testing.assert_allclose(o[h * g.N:(h + 1) * g.N], mean, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[h * g.N:(h + 1) * g.N], np.log(m.sum(1)), rtol=0, atol=1e-12)


def test_one_hot_tile_coordinates_reveal_window_extent():
    """Q = 0 and V = one-hot tile coordinates per dimension: channel c of the
    output is exactly 1/w' for tiles inside the window along that dimension
    and 0 outside, which spells out the window start and length."""
    T, H, W, tile = 10, 12, 16, (2, 3, 4)  # grid 5x4x4
    windows = [(3, 3, 3), (1, 1, 1), (2, 4, 3), (7, 2, 2)]
    g = geom(T, H, W, tile, windows, d=16)
    G = (5, 4, 4)
    v = torch.zeros(1, g.Hh, g.N, g.d)
    for n in range(g.N):
        t, h, w = n // (H * W), (n // W) % H, n % W
        v[:, :, n, t // tile[0]] = 1
        v[:, :, n, G[0] + h // tile[1]] = 1
        v[:, :, n, G[0] + G[1] + w // tile[2]] = 1
    v = v.to(torch.bfloat16)
    q = torch.zeros_like(v)
    o, _ = oracle.forward(g, q, v, v)
    o = o.reshape(g.Hh, g.N, g.d)
    for hd, win in enumerate(windows):
        for n in range(g.N):
            qc = (n // (H * W) // tile[0], (n // W) % H // tile[1], n % W // tile[2])
            base = 0
            for dim in range(3):
                wl = min(win[dim], G[dim])
                s = nearest_start(qc[dim], win[dim], G[dim])
                expect = np.array([1.0 / wl if s <= x < s + wl else 0.0 for x in range(G[dim])])
                np.testing.assert_allclose(o[hd, n, base:base + G[dim]], expect, rtol=0, atol=1e-13)
                base += G[dim]


@pytest.mark.parametrize("case", [SMALL_CASES[0], SMALL_CASES[2], SMALL_CASES[4]])
def test_backward_matches_autograd_of_masked_sdpa(case):
    T, H, W, tile, windows = case
    g = geom(T, H, W, tile, windows, B=2, d=16)
    q, k, v, do = rand_inputs(g, seed=29, with_dout=True)
    masks = [brute_mask(g, h) for h in range(g.Hh)]
    qd, kd, vd = (x.double().requires_grad_() for x in (q, k, v))
    mask = torch.stack([torch.from_numpy(m) for m in masks])[None]
    out = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=1.0 / math.sqrt(g.d))
    (out * do.double()).sum().backward()
    for bh in range(g.B * g.Hh):
        b, h = divmod(bh, g.Hh)
        dq, dk, dv = oracle.backward(g, q, k, v, do, bh)
        np.testing.assert_allclose(dq, qd.grad[b, h].numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, kd.grad[b, h].numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, vd.grad[b, h].numpy(), rtol=0, atol=1e-11)


def test_backward_row_subsets_match_full():
    g = geom(4, 6, 8, (2, 2, 2), [(1, 3, 2), (2, 2, 4)], B=1, d=16)
    q, k, v, do = rand_inputs(g, seed=31, with_dout=True)
    dq, dk, dv = oracle.backward(g, q, k, v, do, 1)
    qr = np.array([0, 5, 47, g.N - 1])
    kr = np.array([3, 20, g.N - 2])
    dq2, dk2, dv2 = oracle.backward(g, q, k, v, do, 1, q_rows=qr, k_rows=kr)
    assert np.array_equal(dq2, dq[qr]) and np.array_equal(dk2, dk[kr]) and np.array_equal(dv2, dv[kr])


def test_backward_finite_differences():
    """Central differences of L = sum(O * dO) in fp64, on a grid small enough
    for a few hundred oracle calls.  Inputs are bf16-representable, and the
    perturbation is applied in fp64 through a float64 copy of the problem."""
    g = geom(2, 4, 4, (1, 2, 2), [(1, 2, 1)], B=1, d=4)  # grid 2x2x2, 32 tokens
    q, k, v, do = rand_inputs(g, seed=37, with_dout=True)
    dq, dk, dv = oracle.backward(g, q, k, v, do, 0)
    # fp64 forward through the oracle's own definition needs bf16 inputs, so
    # the perturbation is done on a masked fp64 replica whose forward values are
    # checked against the oracle first.
    m = torch.from_numpy(brute_mask(g, 0))
    scale = 1.0 / math.sqrt(g.d)

    def loss(qq, kk, vv):
        s = (qq @ kk.T) * scale
        s = s.masked_fill(~m, -math.inf)
        p = torch.exp(s - s.max(-1, keepdim=True).values)
        p = p / p.sum(-1, keepdim=True)
        return ((p @ vv) * do.double()[0, 0]).sum()

    base = [x.double()[0, 0].clone() for x in (q, k, v)]
    o_ref, _ = oracle.forward(g, q, k, v)
    s = (base[0] @ base[1].T) * scale
    s = s.masked_fill(~m, -math.inf)
    np.testing.assert_allclose((torch.softmax(s, -1) @ base[2]).numpy(), o_ref, rtol=0, atol=1e-13)
    eps = 1e-6
    for which, grad in enumerate((dq, dk, dv)):
        for i in range(g.N):
            for c in range(g.d):
                plus = [x.clone() for x in base]
                minus = [x.clone() for x in base]
                plus[which][i, c] += eps
                minus[which][i, c] -= eps
                fd = (loss(*plus) - loss(*minus)).item() / (2 * eps)
                assert abs(fd - grad[i, c]) <= 1e-6 * max(1.0, abs(fd)), (which, i, c, fd, grad[i, c])
