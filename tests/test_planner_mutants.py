"""The planner's tests catch plausible mistakes: each case plants one mistake in
a copy of csrc/sta_api.cpp (window placement, list order, inverse lists, block
pairing, work order and coverage, the host slice groups), links it with the
library's other objects into a libsta.so of its own, and runs
tests/test_plan.py and tests/test_plan_work.py against it (host-only plans,
no GPU).  Every mutant must fail at least one of them; the unmodified source,
built the same way, must pass them all.  No mutant indexes outside the
planner's tables."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from sparse_local_attention_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(_build.CSRC, "sta_api.cpp")

# (name, text in sta_api.cpp, replacement); every occurrence is replaced
MUTANTS = [
    ("window_start_rounds_up", "  int s = q - w / 2;", "  int s = q - (w + 1) / 2;"),
    ("list_order_w_before_h",
     "            for (int kt = st; kt < st + w[0]; ++kt)\n"
     "              for (int kh = sh; kh < sh + w[1]; ++kh)\n"
     "                for (int kw = sw; kw < sw + w[2]; ++kw)",
     "            for (int kt = st; kt < st + w[0]; ++kt)\n"
     "              for (int kw = sw; kw < sw + w[2]; ++kw)\n"
     "                for (int kh = sh; kh < sh + w[1]; ++kh)"),
    ("inverse_lists_descending", "        for (int qtile = 0; qtile < g.n_tiles; ++qtile) {",
     "        for (int qtile = g.n_tiles - 1; qtile >= 0; --qtile) {"),
    ("pairs_ignore_the_t_window",
     "const std::array<int, 3> key = {window_start(qt, w[0], g.GT),",
     "const std::array<int, 3> key = {0 * window_start(qt, w[0], g.GT),"),
    ("lone_blocks_first", "    pl->work.insert(pl->work.end(), lone_items.begin(), lone_items.end());",
     "    pl->work.insert(pl->work.begin(), lone_items.begin(), lone_items.end());"),
    ("forward_cost_ascending", "return cost(a) > cost(b);", "return cost(a) < cost(b);"),
    ("dkdv_shortest_first", "a.bh < c.bh : a.len > c.len;", "a.bh < c.bh : a.len < c.len;"),
    ("dkdv_slices_interleaved", "return a.bh != c.bh ? a.bh < c.bh : a.len > c.len;", "return a.len > c.len;"),
    ("dq_last_block_missing", "            for (int qb = 0; qb < nqb; ++qb) pl->work_q.push_back(",
     "            for (int qb = 0; qb + 1 < nqb || (nqb == 1 && qb < 0); ++qb) pl->work_q.push_back("),
    ("host_groups_shifted", "pl->group_slice[gi] = (int)((long long)slices * gi / groups);",
     "pl->group_slice[gi] = (int)((long long)slices * gi / groups) + (gi > 0 && gi < groups ? 1 : 0);"),
]


def _run(tmp_path, name, text, repl):
    src = open(SRC).read()
    if text is not None:
        assert text in src, f"{name}: pattern not in sta_api.cpp"
        src = src.replace(text, repl)
    cpp = tmp_path / f"{name}.cpp"
    obj = tmp_path / f"{name}.o"
    lib = tmp_path / f"libsta_{name}.so"
    # the copy sits outside csrc/: point its relative include of sta.h at the real header
    cpp.write_text(src.replace('#include "../../include/sta.h"', '#include "sta.h"'))
    cmd = _build.compile_command(str(cpp), str(obj)) + ["-I", _build.CSRC]
    subprocess.run(cmd, check=True, capture_output=True)
    objs = [str(obj) if n == "sta_api.cpp" else o for n, o in _build.objects().items()]
    subprocess.run(_build.link_command(objs, str(lib)), check=True, capture_output=True)
    env = dict(os.environ, STA_LIBRARY=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_plan.py"), os.path.join(ROOT, "tests", "test_plan_work.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True)
    return name, r.returncode, r.stdout[-2000:]


def test_every_planted_planner_mistake_fails_a_test(tmp_path):
    if not os.path.exists(_build.LIB) or any(not os.path.exists(o) for o in _build.objects().values()):
        _build.build()
    cases = [("unmodified", None, None)] + MUTANTS
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda c: _run(tmp_path, *c), cases))
    control = results[0]
    assert control[1] == 0, f"unmodified planner fails its tests:\n{control[2]}"
    survivors = [(name, out) for name, code, out in results[1:] if code != 1]
    assert not survivors, "mutants not caught (pytest exit code != 1):\n" + "\n".join(
        f"{n}:\n{o}" for n, o in survivors)
