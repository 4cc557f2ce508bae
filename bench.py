"""Benchmark: Sliding Tile Attention forward on B200.

Metric: STA forward ms per call and useful TFLOP/s on the 30x48x80 video latent
(24 heads, d=128, tile 6x8x8, window 3x3x3), with useful FLOPs
4 * N * keys_per_query * d per head, and the fraction of the measured dense
BF16 tensor-core peak.  One step = one sta_forward call (the whole hot path:
K/V gather, QK^T, softmax, PV, O/LSE write-back) on inputs resident in HBM.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        python bench.py --impl reference ...   (the fp64 CPU oracle arm)
Multi-GPU: launched by torchrun, one rank per GPU; every rank runs its own
independent problem (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_local_attention_b200.workloads import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "STA fwd ms and useful TFLOPS at 30×48×80, 24 heads, d=128; % of BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "sta_fwd_kernel_dit720p.md")
KERNEL_SOURCE = os.path.join(ROOT, "sparse_local_attention_b200", "csrc", "sta_fwd.cu")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_hash() -> str:
    with open(KERNEL_SOURCE, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes of one forward call (every launch it makes) from the committed
    ncu summary, if it was taken on this workload with the current kernel source."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    txt = open(PROFILE_SUMMARY).read()
    m = re.search(r"traffic_bytes_per_call:\s*([0-9.eE+]+)\s+workload:\s*(\S+)\s+kernel_sha:\s*(\w+)", txt)
    if not m or m.group(2) != workload or m.group(3) != kernel_hash():
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(1.0)  # let nvidia-smi start before the timed region
        return self

    def mark(self, which: str):
        setattr(self, which, time.time())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        import datetime
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "start", None), getattr(self, "stop", None)
        for r in rows:
            r = [x.strip() for x in r]
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if t0 is not None and t1 is not None and not (t0 - 0.05 <= ts <= t1 + 0.05):
                    continue
                sm.append(float(r[2]))
                mx = float(r[3])
            except (ValueError, IndexError):
                continue
            for nm, val in zip(names, r[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    """Process group for barriers and max-over-ranks timing only (the ranks
    share no data).  NCCL on the GPUs; gloo serves the host-side tests."""
    if world > 1:
        import datetime

        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
        return dist
    return None


def max_over_ranks(dist, x: float, device="cuda") -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_share(wl, world: int, rank: int, shard: str):
    """This rank's problem: (workload, heads or None, the job's useful forward
    FLOPs per step, scaling).

    shard "problem": every rank runs the whole workload on inputs seeded by
    its rank (weak scaling: per-GPU work fixed as N grows).  shard "heads":
    the ranks split one problem's heads, longest-processing-time by keys per
    query, and each keeps its heads of the same seeded inputs (strong
    scaling: the job is fixed)."""
    from sparse_local_attention_b200.sharding import head_costs, partition_heads, shard_workload
    if shard == "heads":
        parts = partition_heads(head_costs(wl), world)
        if any(not p for p in parts):
            raise SystemExit(f"--shard heads: {wl.Hh} heads cannot give each of {world} ranks at least one")
        return shard_workload(wl, parts[rank]), parts[rank], wl.forward_flops(), "strong"
    return wl, None, wl.forward_flops() * world, "weak"


def call_stats(per_call_ms):
    """Median, 10th and 90th percentile of per-call times (ms)."""
    p10, p50, p90 = np.percentile(np.asarray(per_call_ms, dtype=np.float64), [10, 50, 90])
    return {"median": float(p50), "p10": float(p10), "p90": float(p90), "calls": len(per_call_ms)}


def timed_leg(fn, warmup: int, steps: int, stream):
    """warmup untimed calls, then steps calls timed with CUDA events on stream:
    {"ms_per_call": mean, "per_call_ms": median / p10 / p90}."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ms, per_call = timed_calls(fn, steps, stream)
    return {"ms_per_call": ms, "per_call_ms": call_stats(per_call), "warmup": warmup, "steps": steps}


def extra_legs(sta, peak: float, peak_source: str, stream, q, k, v, steps: int):
    """The other workloads of the benchmark family, each timed on its own
    inputs (resident in HBM, larger than L2) after 3 warm-up calls:
      backward:     the fine-tuning workload's sta_backward, and its sta_forward;
      perhead:      the per-head-window workload's sta_forward;
      full_window:  the 720p latent with the window = the whole tile grid (dense
                    attention through STA) beside the library's dense SDPA on
                    the same tensors (q, k, v of the headline workload, which
                    are the full-window workload's inputs: same shape, same seed)."""
    def rate(flops, ms):
        t = flops / (ms * 1e-3) / 1e12
        return {"tflops_useful": t, "frac_of_peak": t / peak, "peak_source": peak_source}

    legs = {}
    # --- backward (fine-tuning workload)
    wl = WORKLOADS["finetune"]
    qf, kf, vf, dof = (x.cuda() for x in make_inputs(wl, with_dout=True))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=True))
    of = torch.empty_like(qf)
    lsef = torch.empty(wl.B, wl.Hh, wl.N, dtype=torch.float32, device="cuda")
    fws, bws = plan.workspace(), plan.workspace(backward=True)
    dq, dk, dv = torch.empty_like(qf), torch.empty_like(kf), torch.empty_like(vf)
    sta.sta_forward(plan, qf, kf, vf, of, lsef, fws, stream, check=True)
    sta.sta_backward(plan, qf, kf, vf, of, lsef, dof, dq, dk, dv, bws, stream, check=True)
    fwd = timed_leg(lambda: sta.sta_forward(plan, qf, kf, vf, of, lsef, fws, stream), 3, steps, stream)
    bwd = timed_leg(lambda: sta.sta_backward(plan, qf, kf, vf, of, lsef, dof, dq, dk, dv, bws, stream), 3, steps,
                    stream)
    legs["backward"] = {"workload": f"{wl.name}: {wl.description}", **bwd, **rate(wl.backward_flops(), bwd["ms_per_call"]),
                        "useful_tflop_per_call": wl.backward_flops() / 1e12,
                        "useful_flop_convention": "2.5 x forward (five GEMM-shaped products)",
                        "kernels_per_call": plan.backward_launches,
                        "forward": {**fwd, **rate(wl.forward_flops(), fwd["ms_per_call"]),
                                    "useful_tflop_per_call": wl.forward_flops() / 1e12}}
    plan.destroy()
    del qf, kf, vf, dof, of, lsef, fws, bws, dq, dk, dv
    # --- per-head windows
    wl = WORKLOADS["dit720p_perhead"]
    qp, kp, vp = (x.cuda() for x in make_inputs(wl))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl))
    op = torch.empty_like(qp)
    lsep = torch.empty(wl.B, wl.Hh, wl.N, dtype=torch.float32, device="cuda")
    ws = plan.workspace()
    sta.sta_forward(plan, qp, kp, vp, op, lsep, ws, stream, check=True)
    fwd = timed_leg(lambda: sta.sta_forward(plan, qp, kp, vp, op, lsep, ws, stream), 3, steps, stream)
    legs["perhead"] = {"workload": f"{wl.name}: {wl.description}", **fwd, **rate(wl.forward_flops(), fwd["ms_per_call"]),
                       "useful_tflop_per_call": wl.forward_flops() / 1e12}
    plan.destroy()
    del qp, kp, vp, op, lsep, ws
    # --- full window: dense attention through STA, beside the library's SDPA
    wl = WORKLOADS["dit720p_full"]
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl))
    o = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hh, wl.N, dtype=torch.float32, device="cuda")
    ws = plan.workspace()
    sta.sta_forward(plan, q, k, v, o, lse, ws, stream, check=True)
    fwd = timed_leg(lambda: sta.sta_forward(plan, q, k, v, o, lse, ws, stream), 3, steps, stream)
    sdpa = timed_leg(lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v), 3, steps, stream)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    err = (o.float() - ref.float()).abs()
    legs["full_window"] = {"workload": f"{wl.name}: {wl.description}", **fwd,
                           **rate(wl.forward_flops(), fwd["ms_per_call"]),
                           "useful_tflop_per_call": wl.forward_flops() / 1e12,
                           "sdpa": {"impl": "torch.nn.functional.scaled_dot_product_attention (bf16)", **sdpa,
                                    **rate(wl.forward_flops(), sdpa["ms_per_call"])},
                           "sta_vs_sdpa_max_abs_diff": float(err.max()), "sta_vs_sdpa_mean_abs_diff": float(err.mean())}
    plan.destroy()
    return legs


def timed_calls(fn, steps: int, stream):
    """Run fn steps times between CUDA events on stream, one event after each
    call; return (mean ms over the whole region, per-call ms)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(steps):
        fn()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per_call = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    return evs[0].elapsed_time(evs[-1]) / steps, per_call


# ---------------------------------------------------------------- CPU oracle timing
def oracle_sample_rows(wl, n_rows: int):
    """First n_rows query rows of the first (batch, head) slice, tile by tile
    from the middle of the grid (interior windows)."""
    from sparse_local_attention_b200.workloads import tile_tokens
    rows, tile = [], wl.n_tiles // 2
    while len(rows) < n_rows:
        rows.extend(tile_tokens(wl, tile % wl.n_tiles))
        tile += 1
    return np.array(rows[:n_rows], dtype=np.int64)


def time_oracle(wl, q, k, v, target_s: float):
    """Time the oracle (as it stands) on a bounded sample of the workload and
    return (TFLOP/s, sample description, threads)."""
    import oracle
    g = oracle.Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))
    flops_per_row = 4.0 * wl.keys_per_query(0) * wl.d
    oracle.forward(g, q, k, v, rows=oracle_sample_rows(wl, 64))  # thread pool, input conversion
    n = 1024  # calibration sample
    t0 = time.perf_counter()
    oracle.forward(g, q, k, v, rows=oracle_sample_rows(wl, n))
    dt = time.perf_counter() - t0
    n2 = int(max(n, min(wl.N, n * target_s / max(dt, 1e-3))))
    rows = oracle_sample_rows(wl, n2)
    t0 = time.perf_counter()
    oracle.forward(g, q, k, v, rows=rows)
    dt = time.perf_counter() - t0
    tflops = flops_per_row * len(rows) / dt / 1e12
    cores = oracle.threads()
    # the same rows on one thread, a quarter of the time budget
    n1 = int(max(64, min(len(rows), len(rows) * target_s / 4 / max(dt * cores, 1e-3))))
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.forward(g, q, k, v, rows=rows[:n1])
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(cores)
    extra = {"single_thread_tflops": flops_per_row * n1 / dt1 / 1e12,
             "single_thread_sample": f"{n1} of the same rows, {dt1:.1f} s",
             "extrapolated_full_call_s": wl.forward_flops() / (tflops * 1e12)}
    return tflops, dt, f"{len(rows)} query rows of head 0 ({wl.keys_per_query(0)} keys each), {dt:.1f} s", cores, extra


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    import oracle
    q, k, v = make_inputs(wl)
    g = oracle.Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))
    rows = oracle_sample_rows(wl, args.ref_rows)
    flops = 4.0 * wl.keys_per_query(0) * wl.d * len(rows)
    for _ in range(args.warmup):
        oracle.forward(g, q, k, v, rows=rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(g, q, k, v, rows=rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = f"{len(rows)} query rows of head 0 per step ({wl.keys_per_query(0)} keys each)"
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: {wl.description}", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def run_ours(args):
    from sparse_local_attention_b200 import sta

    from sparse_local_attention_b200.sharding import select_heads

    world, rank, local = dist_env()
    wl_job = WORKLOADS[args.workload]
    wl, heads, job_flops, scaling = rank_share(wl_job, world, rank, args.shard)
    dist = init_dist(world, local)
    torch.cuda.set_device(local)
    pk, pk_kind = peaks()

    def inputs(with_dout=False):
        """This rank's inputs: its own seeded problem, or its heads of the job's."""
        if heads is None:
            return make_inputs(wl, with_dout=with_dout, seed=rank)
        return tuple(select_heads(x, heads) for x in make_inputs(wl_job, with_dout=with_dout, seed=0))

    q_h, k_h, v_h = (x.pin_memory() for x in inputs())
    q, k, v = (x.cuda() for x in (q_h, k_h, v_h))
    plan = sta.sta_plan_create(sta.Problem.from_workload(wl, backward=wl.backward))
    o = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hh, wl.N, dtype=torch.float32, device="cuda")
    ws = plan.workspace()
    stream = torch.cuda.current_stream()

    def step():
        sta.sta_forward(plan, q, k, v, o, lse, ws, stream)

    sta.sta_forward(plan, q, k, v, o, lse, ws, stream, check=True)  # one checked call
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.mark("start")
        ms_rank, per_call = timed_calls(step, args.steps, stream)
        clk.mark("stop")
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, ms_rank)
    flops = wl.forward_flops()  # this rank's
    value = job_flops / (ms * 1e-3) / 1e12
    launches_per_step = plan.forward_launches  # kernels one sta_forward call enqueues

    # --- backward (fine-tuning workloads): dQ, dK, dV from the same inputs
    bwd = None
    if wl.backward:
        do_h = inputs(with_dout=True)[3]
        dout = do_h.cuda()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = plan.workspace(backward=True)
        sta.sta_backward(plan, q, k, v, o, lse, dout, dq, dk, dv, bws, check=True)
        for _ in range(args.warmup):
            sta.sta_backward(plan, q, k, v, o, lse, dout, dq, dk, dv, bws)
        torch.cuda.synchronize()
        bms_rank, bper_call = timed_calls(
            lambda: sta.sta_backward(plan, q, k, v, o, lse, dout, dq, dk, dv, bws), args.steps, stream)
        bms = max_over_ranks(dist, bms_rank)
        bwd = {"ms_per_step": bms, "tflops_useful": 2.5 * job_flops / (bms * 1e-3) / 1e12,
               "per_call_ms_rank0": call_stats(bper_call),
               "useful_flop_convention": "2.5 x forward (five GEMM-shaped products)",
               "kernels_per_step": plan.backward_launches}
        del dout, dq, dk, dv, bws

    # --- permute kernel (raster <-> tile-major, HBM-bound): on the forward path
    #     only when tiles are not TMA boxes of the raster tensor; measured here
    #     on Q of the same workload, both directions
    perm_t = torch.empty_like(q)
    perm_back = torch.empty_like(q)
    for _ in range(3):
        sta.sta_permute(plan, q, perm_t, stream=stream)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    perm_reps = 10
    p0.record(stream)
    for _ in range(perm_reps):
        sta.sta_permute(plan, q, perm_t, stream=stream)
        sta.sta_permute(plan, perm_t, perm_back, inverse=True, stream=stream)
    p1.record(stream)
    torch.cuda.synchronize()
    perm_ms = p0.elapsed_time(p1) / (2 * perm_reps)
    if not torch.equal(perm_back, q):
        raise RuntimeError("permute round trip is not the identity")
    perm_bytes = 2 * q.numel() * q.element_size()  # read + write
    hbm_peak = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    permute = {"kernel": "permute_kernel", "ms_per_launch": perm_ms, "bytes_per_launch": perm_bytes,
               "achieved_gbs": perm_bytes / (perm_ms * 1e-3) / 1e9, "peak_gbs": hbm_peak,
               "frac": perm_bytes / (perm_ms * 1e-3) / 1e9 / hbm_peak,
               "peak_source": f"{pk_kind} hbm_gbs", "bound": "hbm"}
    del perm_t, perm_back

    # --- end to end through the C ABI with host buffers (sta_forward_host):
    #     pinned host Q, K, V in, host O and LSE out; the library copies the
    #     (batch, head) slices in groups and overlaps the copies with the kernels
    o_h = torch.empty_like(q_h).pin_memory()
    lse_h = torch.empty(wl.B, wl.Hh, wl.N, dtype=torch.float32).pin_memory()
    hws = plan.workspace(host=True)

    def e2e_step():
        sta.sta_forward_host(plan, q_h, k_h, v_h, o_h, lse_h, hws, stream)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1) / e2e_steps)
    if not torch.equal(o_h, o.cpu()):
        raise RuntimeError("sta_forward_host output differs from sta_forward")
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4

    # --- dense full-attention baseline on the same shapes (library SDPA)
    dense = None
    if not args.no_dense and rank == 0 and heads is None:
        torch.backends.cuda.enable_flash_sdp(True)
        for _ in range(2):
            torch.nn.functional.scaled_dot_product_attention(q, k, v)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        d0.record(stream)
        for _ in range(reps):
            torch.nn.functional.scaled_dot_product_attention(q, k, v)
        d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / reps
        dflops = 4.0 * wl.N * wl.N * wl.d * wl.Hh * wl.B
        dense = {"impl": "torch.nn.functional.scaled_dot_product_attention (full 3D attention, bf16)",
                 "ms": dms, "tflops": dflops / (dms * 1e-3) / 1e12, "speedup_sta_vs_dense": dms / ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tflops, dt, sample, cores, extra = time_oracle(wl, q_h, k_h, v_h, args.cpu_seconds)
        cpu = {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample, **extra}

    legs = {}
    if rank == 0 and world == 1 and args.workload == HEADLINE and not args.no_extra_legs:
        peak_x = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        legs = extra_legs(sta, peak_x, f"{pk_kind} bf16_tflops", stream, q, k, v, max(10, min(args.steps, 20)))

    clocks = clk.summary()
    if rank == 0:
        peak_key = "bf16_tflops"
        peak = float(pk.get(peak_key, FALLBACK_PEAKS[peak_key]))
        if bwd is not None:
            # the backward's useful rate per GPU against the same measured bf16 peak
            bwd["frac_of_peak"] = bwd["tflops_useful"] / world / peak
            bwd["peak_source"] = f"{pk_kind} {peak_key}"
        achieved = flops / (ms * 1e-3) / 1e12
        traffic = profiled_traffic(wl.name)
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "per_call_ms_rank0": call_stats(per_call),
            "higher_is_better": True, "scaling": scaling,
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{wl_job.name}: {wl_job.description}",
                       "useful_tflop_per_step": job_flops / 1e12, "useful_tflop_per_step_rank0": flops / 1e12,
                       "l2": "inputs 3 x %.0f MB per GPU, larger than the 126 MB L2; no flush" % (q.numel() * 2 / 1e6),
                       "parallelism": (f"independent problem per GPU x{world}" if heads is None else
                                       f"heads split over {world} GPUs by keys per query (rank 0: heads {heads})")},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{pk_kind} {peak_key}",
                         "kernel": "sta_fwd_kernel (one forward call: %d launch(es), timed together)" % launches_per_step,
                         "per": "forward call"},
            "e2e": {"value": job_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "dense_baseline": dense,
            "backward": bwd,
            "permute": permute,
        }
        if legs:
            if out["backward"] is None:
                out["backward"] = legs.pop("backward")
            out.update(legs)
        print(json.dumps(out), flush=True)
    plan.destroy()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-legs", action="store_true",
                    help="skip the backward / per-head / full-window records of the default run")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=384)
    ap.add_argument("--shard", default="problem", choices=["problem", "heads"],
                    help="problem: one independent problem per GPU (weak scaling); "
                         "heads: one problem's heads split over the GPUs (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
