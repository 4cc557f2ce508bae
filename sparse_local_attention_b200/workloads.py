"""Seeded synthetic workloads for Sliding Tile Attention.

This module only describes problem shapes and draws random inputs; it holds no
attention arithmetic, so both the CUDA path's tests and the CPU oracle can use
it.  The latent shape 30x48x80 is the VAE latent of a 720P, 5 s video
("Fast Video Generation with Sliding Tile Attention", summary page,
Experiments).  The pages' real workloads (HunyuanVideo latents) are not
available, so i.i.d. N(0, 1) values (plus, for the per-head case, a smooth 3D
sinusoidal field that makes scores locally peaked) stand in for them.

Recipe: torch.Generator().manual_seed(seed) on the CPU; fp32 N(0, 1) drawn in
the order Q, K, V, dO; the optional field is added; then each tensor is
rounded to bf16 (round-to-nearest-even).  Tensors are [B, heads, N, d] with
token n = (t*H + h)*W + w (raster order).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hh: int
    d: int
    T: int
    H: int
    W: int
    tile: tuple
    windows: tuple  # one (w_t, w_h, w_w) per head, in tiles
    field_amplitude: float = 0.0
    backward: bool = False
    seed: int = 0
    description: str = ""

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def grid(self) -> tuple:
        return (self.T // self.tile[0], self.H // self.tile[1], self.W // self.tile[2])

    @property
    def n_tiles(self) -> int:
        g = self.grid
        return g[0] * g[1] * g[2]

    @property
    def tile_volume(self) -> int:
        return self.tile[0] * self.tile[1] * self.tile[2]

    def keys_per_query(self, head: int) -> int:
        """Keys each query of `head` attends to: whole tiles of the window,
        the window clamped to the tile grid."""
        g = self.grid
        w = self.windows[head]
        n = 1
        for i in range(3):
            n *= min(w[i], g[i])
        return n * self.tile_volume

    def forward_flops(self) -> float:
        """Useful forward FLOPs: 4 * N * keys_per_query * d, per head and batch."""
        return float(sum(4.0 * self.N * self.keys_per_query(h) * self.d for h in range(self.Hh)) * self.B)

    def backward_flops(self) -> float:
        """Useful backward FLOPs: 2.5x the forward (five GEMM-shaped products)."""
        return 2.5 * self.forward_flops()

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload(
        "tiny", B=1, Hh=2, d=64, T=6, H=16, W=16, tile=(2, 4, 4), windows=((3, 3, 3),) * 2,
        description="1x2 heads, d64, latent 6x16x16 (1536 tokens), tile 2x4x4, window 3x3x3"),
    "dit720p": Workload(
        "dit720p", B=1, Hh=24, d=128, T=30, H=48, W=80, tile=(6, 8, 8), windows=((3, 3, 3),) * 24,
        description="1x24 heads, d128, latent 30x48x80 (115200 tokens), tile 6x8x8, window 3x3x3"),
    "dit720p_perhead": Workload(
        "dit720p_perhead", B=1, Hh=24, d=128, T=30, H=48, W=80, tile=(6, 8, 8),
        windows=((1, 3, 3),) * 8 + ((3, 3, 5),) * 8 + ((5, 5, 5),) * 8, field_amplitude=1.0,
        description="1x24 heads, d128, latent 30x48x80, tile 6x8x8, per-head windows "
                    "1x3x3 / 3x3x5 / 5x5x5, N(0,1) + sinusoidal field"),
    "dit720p_full": Workload(
        "dit720p_full", B=1, Hh=24, d=128, T=30, H=48, W=80, tile=(6, 8, 8), windows=((5, 6, 10),) * 24,
        description="1x24 heads, d128, latent 30x48x80, tile 6x8x8, window 5x6x10 = whole grid"),
    "finetune": Workload(
        "finetune", B=2, Hh=16, d=64, T=16, H=64, W=64, tile=(4, 8, 8), windows=((3, 5, 5),) * 16,
        backward=True,
        description="2x16 heads, d64, latent 16x64x64 (65536 tokens), tile 4x8x8, window 3x5x5, fwd+bwd"),
}

HEADLINE = "dit720p"


def positional_field(wl: Workload, seed: int = 1) -> torch.Tensor:
    """Smooth 3D sinusoidal field F[n, c] of amplitude wl.field_amplitude.

    F[t,h,w,c] = A * sin(2*pi*(a_c*t/T + b_c*h/H + e_c*w/W) + phi_c), with
    integers a_c, b_c, e_c uniform in {1..4} and phi_c uniform in [0, 2*pi),
    drawn from a generator seeded with `seed`."""
    g = torch.Generator().manual_seed(seed)
    a = torch.randint(1, 5, (wl.d,), generator=g).double()
    b = torch.randint(1, 5, (wl.d,), generator=g).double()
    e = torch.randint(1, 5, (wl.d,), generator=g).double()
    phi = torch.rand(wl.d, generator=g).double() * (2 * math.pi)
    t = torch.arange(wl.T).double().view(-1, 1, 1, 1) / wl.T
    h = torch.arange(wl.H).double().view(1, -1, 1, 1) / wl.H
    w = torch.arange(wl.W).double().view(1, 1, -1, 1) / wl.W
    f = wl.field_amplitude * torch.sin(2 * math.pi * (a * t + b * h + e * w) + phi)
    return f.reshape(wl.N, wl.d).float()


def make_inputs(wl: Workload, with_dout: bool = False, seed: int | None = None):
    """(q, k, v[, dout]) as bf16 CPU tensors [B, Hh, N, d], drawn as documented above."""
    g = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    shape = (wl.B, wl.Hh, wl.N, wl.d)
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    fld = positional_field(wl) if wl.field_amplitude else None
    out = []
    for nm in names:
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if fld is not None and nm != "dout":
            x += fld
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def tiles_sample(wl: Workload, n: int = 64, seed: int = 0) -> list:
    """Seeded sample of query-tile indices (tile-major order, t outer, w inner):
    the 8 corner tiles of the grid, then seeded random others, n in total."""
    gt, gh, gw = wl.grid
    corners = sorted({(t * gh + h) * gw + w for t in (0, gt - 1) for h in (0, gh - 1) for w in (0, gw - 1)})
    if n >= wl.n_tiles:
        return list(range(wl.n_tiles))
    g = torch.Generator().manual_seed(seed)
    rest = [int(i) for i in torch.randperm(wl.n_tiles, generator=g) if int(i) not in corners]
    return sorted(corners + rest[: max(0, n - len(corners))])


def tile_tokens(wl: Workload, tile_index: int) -> list:
    """Raster token indices of one tile, in in-tile row-major order (t, h, w)."""
    gt, gh, gw = wl.grid
    tt, th, tw = wl.tile
    it, ih, iw = tile_index // (gh * gw), (tile_index // gw) % gh, tile_index % gw
    out = []
    for a in range(tt):
        for b in range(th):
            for c in range(tw):
                t, h, w = it * tt + a, ih * th + b, iw * tw + c
                out.append((t * wl.H + h) * wl.W + w)
    return out
