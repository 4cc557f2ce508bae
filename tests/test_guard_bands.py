"""No writes outside the buffers a call owns (a stand-in for a memory checker).

Every output tensor and the workspace is carved out of a larger allocation
whose bands before and after it are filled with a fixed bit pattern.  After a
checked forward and backward call the bands must still hold the pattern, and
the inputs must be unchanged: a kernel that wrote past a row, a tile, an LSE
run or the workspace would change them.  Ragged tiles (partial 128-row
blocks), the permute fallback and both head dims are covered."""
import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

BAND_BYTES = 64 * 1024  # keeps the carved views 16-byte (and 256-byte) aligned
PATTERN = 0xFF  # all-ones bytes: NaN as bf16 and as fp32


def _guarded(shape, dtype):
    """(whole allocation, contiguous view of `shape` in its middle), every byte
    set to PATTERN."""
    n = 1
    for s in shape:
        n *= s
    elem = torch.empty(0, dtype=dtype).element_size()
    whole = torch.full((2 * BAND_BYTES + n * elem,), PATTERN, dtype=torch.uint8, device="cuda")
    view = whole[BAND_BYTES: BAND_BYTES + n * elem].view(dtype).view(shape)
    return whole, view


def _bands_intact(whole, name):
    lo, hi = whole[:BAND_BYTES], whole[-BAND_BYTES:]
    assert bool((lo == PATTERN).all()), f"{name}: write before the buffer"
    assert bool((hi == PATTERN).all()), f"{name}: write after the buffer"


CASES = {
    "tiny_d64": WORKLOADS["tiny"].with_(backward=True),
    "d128_partial_block": Workload("g1", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3)), backward=True),
    "d64_three_blocks_batch2": Workload("g2", 2, 1, 64, 12, 16, 16, (6, 8, 8), ((3, 3, 3),), backward=True),
    "d128_permute_fallback": Workload("g3", 1, 2, 128, 4, 12, 8, (2, 6, 4), ((3, 1, 2), (2, 2, 2)), backward=True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_calls_write_only_their_outputs_and_workspace(name):
    wl = CASES[name]
    q, k, v, do = (x.cuda() for x in make_inputs(wl, with_dout=True, seed=11))
    copies = [x.clone() for x in (q, k, v, do)]
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    shape = (wl.B, wl.Hh, wl.N, wl.d)
    o_all, o = _guarded(shape, torch.bfloat16)
    l_all, lse = _guarded(shape[:3], torch.float32)
    fw_all, fws = _guarded((plan.fwd_workspace_bytes,), torch.uint8)
    sta.sta_forward(plan, q, k, v, o, lse, fws, check=True)
    grads = [_guarded(shape, torch.bfloat16) for _ in range(3)]
    bw_all, bws = _guarded((plan.bwd_workspace_bytes,), torch.uint8)
    sta.sta_backward(plan, q, k, v, o, lse, do, *(g[1] for g in grads), bws, check=True)
    torch.cuda.synchronize()
    for whole, nm in [(o_all, "o"), (l_all, "lse"), (fw_all, "forward workspace"), (bw_all, "backward workspace")] + \
            [(g[0], n) for g, n in zip(grads, ("dq", "dk", "dv"))]:
        _bands_intact(whole, nm)
    for a, b, nm in zip((q, k, v, do), copies, ("q", "k", "v", "do")):
        assert torch.equal(a, b), f"{nm} was modified"
    # every output element was written: the buffers started as NaN, which
    # finite inputs never produce
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    for g, n in zip(grads, ("dq", "dk", "dv")):
        assert torch.isfinite(g[1]).all(), n
    plan.destroy()
