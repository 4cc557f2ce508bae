"""Per-kernel resources as ptxas reports them (-Xptxas -v), no GPU needed.

A guard against silent regressions of the kernels' register budgets: the
forward and permute kernels run without register spills, and every kernel
fits the registers its launch allows (65536 per SM shared by the block's
warps, allocated per sub-partition: at most 168 per thread for 320 threads,
96 for 576)."""
import os
import re
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

from sparse_local_attention_b200 import _build

KERNELS = ("sta_fwd_kernel", "permute_kernel", "bwd_pre_kernel", "bwd_dq_kernel",
           "bwd_dkdv_kernel")


def _resources(tmp_path):
    """{(kernel, instantiation signature): (registers, spill bytes)} of every kernel."""
    nvcc = _build._nvcc()
    if shutil.which(nvcc) is None and not os.path.exists(nvcc):
        pytest.skip("nvcc not available")

    def one(src):
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xptxas", "-v",
               "-I", os.path.join(_build.ROOT, "include"), "-c", src, "-o", str(tmp_path / (os.path.basename(src) + ".o"))]
        return subprocess.run(cmd, capture_output=True, text=True, check=True).stderr

    with ThreadPoolExecutor(max_workers=4) as ex:
        logs = list(ex.map(one, [s for s in _build.sources() if s.endswith(".cu")]))
    out, current = {}, None
    for line in "\n".join(logs).splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        if current is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            out.setdefault(current, {})["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out.setdefault(current, {})["regs"] = int(m.group(1))
    named = {}
    for mangled, r in out.items():
        for k in KERNELS:
            if re.search(r"\d" + k + r"(I|E)", mangled):
                named.setdefault(k, []).append((mangled, r["regs"], r.get("spill", 0)))
    return named


def test_kernel_register_budgets(tmp_path):
    res = _resources(tmp_path)
    for k in KERNELS:
        assert k in res, f"{k}: no ptxas report"
    for k in ("sta_fwd_kernel", "permute_kernel", "bwd_pre_kernel", "bwd_dq_kernel", "bwd_dkdv_kernel"):
        for mangled, regs, spill in res[k]:
            assert spill == 0, f"{k} ({mangled}) spills {spill} bytes"
    for mangled, regs, spill in res["sta_fwd_kernel"]:
        assert regs <= 168, (mangled, regs)
    for mangled, regs, spill in res["bwd_dkdv_kernel"] + res["bwd_dq_kernel"]:
        # head dim 64 runs 576 threads (96 registers), head dim 128 320 (168)
        cap = 96 if "ILi64E" in mangled else 168
        assert regs <= cap, (mangled, regs)


