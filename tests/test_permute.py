"""Tile-major permutation kernel: bit-exact against a CPU gather."""
import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu


def cpu_tile_major_index(wl: Workload) -> torch.Tensor:
    """src raster token of every tile-major position (tiles t-outer / w-inner,
    tokens inside a tile t-outer / w-inner)."""
    tt, th, tw = wl.tile
    gt, gh, gw = wl.grid
    t = torch.arange(wl.T).view(-1, 1, 1)
    h = torch.arange(wl.H).view(1, -1, 1)
    w = torch.arange(wl.W).view(1, 1, -1)
    tile = ((t // tt) * gh + h // th) * gw + w // tw
    inner = ((t % tt) * th + h % th) * tw + w % tw
    pos = (tile * (tt * th * tw) + inner).reshape(-1)  # position of raster token n
    src = torch.empty_like(pos)
    src[pos] = torch.arange(wl.N)
    return src


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"], WORKLOADS["finetune"], WORKLOADS["dit720p"],
                                Workload("x", 2, 3, 64, 4, 12, 8, (2, 6, 4), ((1, 1, 1),) * 3)],
                         ids=lambda w: w.name)
def test_permute_bit_exact_and_roundtrip(wl):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(wl.B, wl.Hh, wl.N, wl.d, generator=g).to(torch.bfloat16)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    xd = x.cuda()
    y = sta.sta_permute(plan, xd)
    back = sta.sta_permute(plan, y, inverse=True)
    torch.cuda.synchronize()
    idx = cpu_tile_major_index(wl)
    assert torch.equal(y.cpu(), x[:, :, idx])
    assert torch.equal(back, xd)
