"""The N > 1 path of bench.py on the host: two gloo ranks on the CPU (no GPU,
no data-path collective).  Checks max-over-ranks timing, the whole-job rate,
per-rank seeds and that the reference arm runs on rank 0 only; also the
bench's host-side statistics and the oracle timing's thread switch."""
import contextlib
import io
import os
import socket
import sys

import torch
import torch.multiprocessing as mp

from sparse_local_attention_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from sparse_local_attention_b200.workloads import WORKLOADS, make_inputs

    w, r, local = bench.dist_env()
    dist = bench.init_dist(w, local, backend="gloo")
    try:
        # each rank times its own problem; the job's time is the slowest rank's
        ms = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, device="cpu")
        _, _, job_flops, _ = bench.rank_share(WORKLOADS["tiny"], w, r, "problem")
        rate = job_flops / (ms * 1e-3)
        # one problem's heads split over the ranks: every head on exactly one rank
        sub, heads, job_h, scaling = bench.rank_share(WORKLOADS["dit720p_perhead"], w, r, "heads")
        mine = torch.zeros(24)
        mine[heads] = 1.0
        dist.all_reduce(mine)
        # ranks draw different inputs (independent problems)
        q = make_inputs(WORKLOADS["tiny"], seed=r)[0]
        first = torch.tensor([float(q.float().sum())])
        gathered = [torch.zeros(1) for _ in range(w)]
        dist.all_gather(gathered, first)
        # the reference arm: rank 0 only, the others return 0 without output
        out = io.StringIO()
        if r != 0:
            with contextlib.redirect_stdout(out):
                code = bench.run_reference(None)
        else:
            code = 0
        dist.barrier()
        results[rank] = (w, r, ms, rate, [float(x) for x in gathered], code, out.getvalue(),
                         mine.tolist(), sub.forward_flops(), job_h, scaling)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world, start_method="spawn", join=True)
    assert sorted(results.keys()) == [0, 1]
    for rank in range(world):
        w, r, ms, rate, gathered, code, out, cover, sub_flops, job_h, scaling = results[rank]
        assert (w, r) == (world, rank)
        assert ms == 15.0                       # max over ranks, same on every rank
        tiny = WORKLOADS["tiny"].forward_flops()
        assert rate == tiny * world / 15e-3     # all ranks' units over the slowest time
        assert cover == [1.0] * 24              # each head on exactly one rank
        full = WORKLOADS["dit720p_perhead"].forward_flops()
        assert job_h == full and scaling == "strong"
        assert sub_flops == full / world        # three window classes split evenly
        assert gathered[0] != gathered[1]       # per-rank seeds
        assert code == 0 and out == ""


def test_call_stats_percentiles():
    """Per-call statistics in the bench line: median and the 10th / 90th
    percentiles (linear interpolation between order statistics)."""
    sys.path.insert(0, ROOT)
    import bench
    st = bench.call_stats([5.0, 1.0, 3.0, 2.0, 4.0])
    assert st["median"] == 3.0 and st["calls"] == 5
    assert abs(st["p10"] - 1.4) < 1e-12 and abs(st["p90"] - 4.6) < 1e-12


def test_oracle_thread_count_does_not_change_results():
    """The bench times the oracle on all cores and on one; the result must not
    depend on the thread count."""
    import numpy as np
    import oracle
    from sparse_local_attention_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"]
    q, k, v = make_inputs(wl)[:3]
    g = oracle.Geometry(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows))
    rows = np.arange(0, wl.N, 7, dtype=np.int64)
    cores = oracle.threads()
    o_all, lse_all = oracle.forward(g, q, k, v, rows=rows)
    oracle.set_threads(1)
    try:
        assert oracle.threads() == 1
        o_one, lse_one = oracle.forward(g, q, k, v, rows=rows)
    finally:
        oracle.set_threads(cores)
    assert oracle.threads() == cores
    assert np.array_equal(o_all, o_one) and np.array_equal(lse_all, lse_one)
