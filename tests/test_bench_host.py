"""bench.py's own logic on the host: run_ours end to end with the device and
the library replaced by fakes (no GPU), so the JSON line's contract keys and
the forward / backward / head-sharding branches are exercised on every CPU
run.  The numbers are meaningless here; only the structure is checked."""
import argparse
import json
import os
import sys
import time
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_local_attention_b200 import sta  # noqa: E402
from sparse_local_attention_b200.workloads import WORKLOADS  # noqa: E402


class _Event:
    def __init__(self, *a, **k):
        self.t = None

    def record(self, stream=None):
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


class _Plan:
    forward_launches, backward_launches = 2, 3

    def workspace(self, **kw):
        return torch.zeros(16, dtype=torch.uint8)

    def destroy(self):
        pass


class _Clocks:
    def __init__(self, *a):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass

    def mark(self, which):
        pass

    def summary(self):
        return {"sm_mhz": 1.0, "sm_max_mhz": 1.0, "reasons": [], "samples": 0}


@pytest.fixture
def fake_device(monkeypatch):
    empty = torch.empty

    def host_empty(*a, **k):
        k.pop("device", None)
        k.pop("pin_memory", None)
        return empty(*a, **k)

    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: types.SimpleNamespace(cuda_stream=0))
    monkeypatch.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    monkeypatch.setattr(torch, "empty", host_empty)
    monkeypatch.setattr(sta, "sta_plan_create", lambda problem: _Plan())

    def forward(plan, q, k, v, o=None, lse=None, ws=None, stream=None, check=False, want_lse=True):
        o.zero_()
        return o, lse

    def permute(plan, src, dst=None, inverse=False, stream=None):
        dst.copy_(src)
        return dst

    def forward_host(plan, q, k, v, o, lse, ws, stream=None, check=False):
        o.zero_()
        return o, lse

    monkeypatch.setattr(sta, "sta_forward", forward)
    monkeypatch.setattr(sta, "sta_backward", lambda plan, q, k, v, o, lse, do, dq, dk, dv, ws, check=False: (dq, dk, dv))
    monkeypatch.setattr(sta, "sta_permute", permute)
    monkeypatch.setattr(sta, "sta_forward_host", forward_host)
    monkeypatch.setattr(bench, "ClockSampler", _Clocks)
    monkeypatch.setitem(WORKLOADS, "tiny_bwd", WORKLOADS["tiny"].with_(name="tiny_bwd", backward=True))


CONTRACT = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"}


@pytest.mark.parametrize("workload,shard,dense,cpu", [("tiny", "problem", True, False),
                                                     ("tiny_bwd", "problem", False, True),
                                                     ("tiny", "heads", False, False)])
def test_run_ours_prints_the_contract_line(fake_device, capsys, workload, shard, dense, cpu):
    args = argparse.Namespace(gpus=1, steps=4, warmup=3, impl="ours", workload=workload, no_dense=not dense,
                              no_cpu_baseline=not cpu, cpu_seconds=0.2, ref_rows=64, shard=shard)
    assert bench.run_ours(args) == 0
    line = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")][-1]
    d = json.loads(line)
    assert CONTRACT <= set(d)
    assert d["steps"] == 4 and d["gpu_launches"] == 2 * 4
    assert d["scaling"] == ("strong" if shard == "heads" else "weak")
    assert set(d["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert set(d["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert d["e2e"]["h2d_bytes_per_step"] == 3 * WORKLOADS["tiny"].N * 64 * 2 * 2
    assert set(d["per_call_ms_rank0"]) == {"median", "p10", "p90", "calls"}
    assert (d["dense_baseline"] is not None) == dense
    if cpu:
        assert {"value", "unit", "cores", "kind", "sample", "single_thread_tflops",
                "extrapolated_full_call_s"} <= set(d["cpu_baseline"])
    else:
        assert d["cpu_baseline"] is None
    if workload == "tiny_bwd":
        assert {"ms_per_step", "tflops_useful", "frac_of_peak", "kernels_per_step"} <= set(d["backward"])
    else:
        assert d["backward"] is None
