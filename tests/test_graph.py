"""The C ABI's calls capture into a CUDA graph: sta_forward and sta_backward
only enqueue kernels on the caller's stream (no allocation, no host
synchronisation unless STA_CALL_CHECK is given), so a forward + backward step
records once and replays with results bit-identical to eager calls."""
import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"].with_(backward=True),
                                Workload("graph_d128", 1, 2, 128, 8, 8, 8, (4, 4, 4), ((1, 1, 1), (3, 3, 3)),
                                         backward=True)],
                         ids=lambda w: w.name)
def test_forward_and_backward_replay_from_a_cuda_graph(wl):
    q, k, v, do = (x.cuda() for x in make_inputs(wl, with_dout=True, seed=7))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    # eager reference (its first calls also set the kernels' attributes)
    o_ref, lse_ref = sta.sta_forward(plan, q, k, v, check=True)
    g_ref = sta.sta_backward(plan, q, k, v, o_ref, lse_ref, do, check=True)
    o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    fws, bws = plan.workspace(), plan.workspace(backward=True)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        sta.sta_forward(plan, q, k, v, o, lse, fws)
        sta.sta_backward(plan, q, k, v, o, lse, do, dq, dk, dv, bws)
    for _ in range(2):
        for t in (o, lse, dq, dk, dv):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        for name, a, b in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
            assert torch.equal(a, b), name
    del graph
    plan.destroy()
