"""Failure detection without a GPU fault: every barrier wait in the kernels is
bounded.  With the wait limit set to zero the first wait that is not already
satisfied runs out; the kernel records the error, drains its own copies and
MMAs, frees its tensor memory and returns.  The host reports STA_ERR_TIMEOUT
and the CUDA context stays usable: the next call with the normal limit gives
the right answer."""
import pytest
import torch

from sparse_local_attention_b200 import sta
from sparse_local_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_forward_wait_timeout_is_reported_and_recoverable():
    wl = WORKLOADS["tiny"]
    q, k, v = (x.cuda() for x in make_inputs(wl))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    good, _ = sta.sta_forward(plan, q, k, v, check=True)
    try:
        sta.sta_set_wait_limit_ns(0)
        with pytest.raises(sta.StaError) as e:
            sta.sta_forward(plan, q, k, v, check=True)
        assert e.value.status == 8
    finally:
        sta.sta_set_wait_limit_ns(2_000_000_000)
    again, _ = sta.sta_forward(plan, q, k, v, check=True)
    torch.cuda.synchronize()
    assert torch.equal(again, good)


def test_host_forward_wait_timeout_is_reported_and_recoverable():
    """Same through sta_forward_host: the status word of the pipelined call
    reports the time-out, and the next call still gives the device result."""
    wl = WORKLOADS["finetune"].with_(B=1, Hh=4)  # 4 slices in 4 groups
    q, k, v = make_inputs(wl)
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=False))
    good, _ = sta.sta_forward(plan, q.cuda(), k.cuda(), v.cuda(), check=True)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    try:
        sta.sta_set_wait_limit_ns(0)
        with pytest.raises(sta.StaError) as e:
            sta.sta_forward_host(plan, qh, kh, vh, check=True)
        assert e.value.status == 8
    finally:
        sta.sta_set_wait_limit_ns(2_000_000_000)
    again, _ = sta.sta_forward_host(plan, qh, kh, vh, check=True)
    torch.cuda.synchronize()
    assert torch.equal(again, good.cpu())
