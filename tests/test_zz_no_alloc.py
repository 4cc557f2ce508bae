"""sta_backward_noalloc: the backward pass for callers that cannot allocate
device memory where they call it (the whole device already belongs to another
allocator, or the footprint must stay fixed after set-up), so they cannot pass
a workspace.  Its temporaries live in a fixed 32 MiB device array inside
libsta.so.  Two calls in a row, through the C ABI, must match the ordinary
sta_backward (which gets a caller workspace) and the fp64 oracle within the
backward tolerance, and the second call must not change how much device memory
is in use.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes both alone in a
fresh process and after the rest of the suite."""
import numpy as np
import pytest
import torch

import oracle
from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3

CASES = [
    WORKLOADS["tiny"].with_(backward=True),
    Workload("d128", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3)), backward=True),
    # 2x6x4 tiles are not TMA boxes of the raster tensors: Q, K, V and dO are
    # first gathered tile-major into the scratch array, after LSE and D
    Workload("gather", 1, 2, 128, 4, 12, 8, (2, 6, 4), ((3, 1, 2), (2, 2, 2)), backward=True),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_noalloc_backward_matches_workspace_backward(wl):
    q, k, v, do = (x.cuda() for x in make_inputs(wl, with_dout=True, seed=3))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    assert plan.bwd_workspace_bytes <= 32 << 20
    o, lse = sta.sta_forward(plan, q, k, v, check=True)
    ref = sta.sta_backward(plan, q, k, v, o, lse, do, check=True)
    g = oracle.Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))
    exact = [oracle.backward(g, q, k, v, do, bh) for bh in range(wl.B * wl.Hh)]
    outs = [torch.empty_like(q) for _ in range(3)]
    torch.cuda.synchronize()
    for call in range(2):  # the shared scratch keeps the previous call's contents
        for t in outs:
            t.fill_(float("nan"))
        torch.cuda.synchronize()
        used, free = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        got = sta.sta_backward_noalloc(plan, q, k, v, o, lse, do, *outs, check=True)
        torch.cuda.synchronize()
        if call == 1:  # the first call may still load the kernels' code
            assert torch.cuda.memory_allocated() == used
            assert torch.cuda.mem_get_info()[0] == free
        for i, (name, a, b) in enumerate(zip(("dq", "dk", "dv"), got, ref)):
            assert torch.isfinite(a).all(), (call, name)
            err = (a.double() - b.double()).abs()
            assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, name, err.max().item())
            for bh in range(wl.B * wl.Hh):
                e = np.abs(a[bh // wl.Hh, bh % wl.Hh].double().cpu().numpy() - exact[bh][i])
                assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (call, name, bh, e.max())
    plan.destroy()


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 8 x 16 heads x 65536 tokens: LSE and D alone need 2 x 8 x 16 x (65536 + 128) x 4 bytes > 32 MiB
    wl = WORKLOADS["finetune"].with_(B=8)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    assert plan.bwd_workspace_bytes > 32 << 20
    st = sta.lib().sta_backward_noalloc(plan.handle, *([None] * 9), None, 0)
    assert st == 5  # STA_ERR_WORKSPACE, before any pointer is looked at
    plan.destroy()
