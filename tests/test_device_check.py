"""Compute calls run on the calling thread's current device, and a plan's tables
live on the device that was current when it was created.  A call made while
another device is current must be refused on the host with
STA_ERR_INVALID_ARG before anything is enqueued.

A machine with one GPU cannot make another device current, so these tests
build the plan with STA_PROBLEM_DEVICE_CHECK_TEST: its tables are uploaded as
usual, but it records a device number that is never current.  Every compute
call through the C ABI must then fail, and no output, workspace or scratch
byte may change."""
import ctypes

import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

WL = Workload("devcheck", 1, 2, 64, 4, 8, 8, (2, 4, 4), ((3, 3, 3), (1, 1, 1)), backward=True)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_every_compute_call_refuses_a_plan_of_another_device():
    prob = sta.Problem.from_workload(WL, backward=True)
    prob.extra_flags = sta.STA_PROBLEM_DEVICE_CHECK_TEST
    plan = sta.sta_plan_create(prob)
    q, k, v, do = (x.cuda() for x in make_inputs(WL, with_dout=True, seed=11))
    outs = [torch.full_like(q, 7.0) for _ in range(4)]  # o, dq, dk, dv
    lse = torch.full(q.shape[:3], 7.0, dtype=torch.float32, device="cuda")
    ws = torch.full((max(plan.bwd_workspace_bytes, plan.fwd_workspace_bytes),), 0xAB, dtype=torch.uint8,
                    device="cuda")
    hws = torch.full((plan.host_workspace_bytes,), 0xAB, dtype=torch.uint8, device="cuda")
    before = [t.clone() for t in outs + [lse, ws, hws]]
    o, dq, dk, dv = outs
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = sta.lib()
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    oh = torch.full(q.shape, 7.0, dtype=torch.bfloat16).pin_memory()
    lh = torch.full(q.shape[:3], 7.0, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    for flags in (0, sta.STA_CALL_CHECK):
        assert L.sta_forward(plan.handle, _p(q), _p(k), _p(v), _p(o), _p(lse), _p(ws), ws.numel(), stream,
                             flags) == 1
        assert L.sta_backward(plan.handle, _p(q), _p(k), _p(v), _p(o), _p(lse), _p(do), _p(dq), _p(dk), _p(dv),
                              _p(ws), ws.numel(), stream, flags) == 1
        assert L.sta_backward_noalloc(plan.handle, _p(q), _p(k), _p(v), _p(o), _p(lse), _p(do), _p(dq), _p(dk),
                                      _p(dv), stream, flags) == 1
        assert L.sta_forward_host(plan.handle, _p(qh), _p(kh), _p(vh), _p(oh), _p(lh), _p(hws), hws.numel(),
                                  stream, flags) == 1
    assert L.sta_permute(plan.handle, _p(q), _p(o), 0, stream) == 1
    torch.cuda.synchronize()
    for a, b in zip(outs + [lse, ws, hws], before):
        assert torch.equal(a, b)
    assert bool((oh == 7.0).all()) and bool((lh == 7.0).all())
    # through the binding, which makes the current device (the one the plan was
    # created on) current again: the library still refuses the call
    with pytest.raises(sta.StaError) as e:
        sta.sta_forward(plan, q, k, v, o, lse, ws)
    assert e.value.status == 1
    plan.destroy()


def test_noalloc_refuses_a_plan_without_backward_tables():
    """A forward-only plan is an invalid argument for sta_backward_noalloc,
    as for sta_backward, and nothing is written."""
    plan = sta.sta_plan_create(sta.Problem.from_workload(WL, backward=False))
    q, k, v, do = (x.cuda() for x in make_inputs(WL, with_dout=True, seed=12))
    o, lse = sta.sta_forward(plan, q, k, v, check=True)
    grads = [torch.full_like(q, 7.0) for _ in range(3)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = sta.lib().sta_backward_noalloc(plan.handle, _p(q), _p(k), _p(v), _p(o), _p(lse), _p(do),
                                        *(_p(g) for g in grads), stream, sta.STA_CALL_CHECK)
    assert st == 1
    torch.cuda.synchronize()
    assert all(bool((g == 7.0).all()) for g in grads)
    plan.destroy()
