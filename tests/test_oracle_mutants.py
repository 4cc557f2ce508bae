"""The oracle's pins catch plausible mistakes: each case plants one mistake in
a copy of oracle/sta_oracle.c (a dropped term, a wrong sign, a wrong index or
operand, an off-by-one in the window placement), builds it, and runs the pins
of tests/test_oracle.py against that library.  Every mutant must fail at least
one pin other than the two comparisons with torch's masked attention and its
autograd (closed forms, the nearest-centre mask, invariances, the special cases
that reduce to unmasked attention, finite differences), so the oracle stays
pinned even without those; the unmodified source, built the same way, must
pass every pin.

Mistakes are planted in the oracle only, on the CPU.  None of them makes the
oracle read outside its buffers."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sta_oracle.c")

# (name, text in sta_oracle.c, replacement); every occurrence is replaced
MUTANTS = [
    ("window_not_shifted_in_at_far_border", "  if (s > G - w) s = G - w;\n", ""),
    ("window_start_rounds_up", "  int s = qtile - w / 2;", "  int s = qtile - (w + 1) / 2;"),
    ("membership_tests_query_h_tile", "  if (kh / g->th < s || kh / g->th >= s + l) return 0;",
     "  if (qh / g->th < s || qh / g->th >= s + l) return 0;"),
    ("scale_dropped", "    s *= scale;\n", ""),
    ("lse_without_max", "  *lse = m + log(l);", "  *lse = log(l);"),
    ("output_not_normalised", "    const double p = sbuf[j] / l;", "    const double p = sbuf[j];"),
    ("keys_as_values", "    const uint16_t *vrow = v + (bh * g->N + keys[j]) * d;",
     "    const uint16_t *vrow = k + (bh * g->N + keys[j]) * d;"),
    ("bf16_low_bit_lost", "  uint32_t u = (uint32_t)b << 16;", "  uint32_t u = (uint32_t)(b & 0xFFFEu) << 16;"),
    ("d_from_dout_dout", "        for (int c = 0; c < d; ++c) s += widen(dorow[c]) * o[c];",
     "        for (int c = 0; c < d; ++c) s += widen(dorow[c]) * widen(dorow[c]);"),
    ("ds_sign", "const double ds = p * (dp - dd[i]);", "const double ds = p * (dp + dd[i]);"),
    ("dq_from_queries", "        for (int c = 0; c < d; ++c) out[c] += scale * ds * widen(krow[c]);",
     "        for (int c = 0; c < d; ++c) out[c] += scale * ds * widen(qrow[c]);"),
    ("dk_without_scale", "        odk[c] += scale * ds * widen(qrow[c]);", "        odk[c] += ds * widen(qrow[c]);"),
    ("dv_from_ds", "        odv[c] += p * widen(dorow[c]);", "        odv[c] += ds * widen(dorow[c]);"),
    ("backward_p_without_scale", "const double p = exp(scale * s - lse[i]);", "const double p = exp(s - lse[i]);"),
]


INDEPENDENT = "not sdpa and not autograd"  # every pin but the two masked-attention comparisons


def _run_pins(tmp_path, name, text, repl):
    src = open(SRC).read()
    if text is not None:
        assert text in src, f"{name}: pattern not in the oracle source"
        src = src.replace(text, repl)
    c_file = tmp_path / f"{name}.c"
    so_file = tmp_path / f"lib_{name}.so"
    c_file.write_text(src)
    subprocess.run(oracle.compile_command(str(c_file), str(so_file)), check=True, capture_output=True)
    env = dict(os.environ, STA_ORACLE_LIB=str(so_file), OMP_NUM_THREADS="2")
    select = [] if text is None else ["-k", INDEPENDENT]  # the control runs every pin
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"), "-x", "-q",
                        "-p", "no:cacheprovider", *select], cwd=ROOT, env=env, capture_output=True, text=True)
    return name, r.returncode, r.stdout[-2000:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    cases = [("unmodified", None, None)] + MUTANTS
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda c: _run_pins(tmp_path, *c), cases))
    control = results[0]
    assert control[1] == 0, f"unmodified oracle fails its pins:\n{control[2]}"
    survivors = [(name, out) for name, code, out in results[1:] if code != 1]
    assert not survivors, "mutants not caught (pytest exit code != 1):\n" + "\n".join(
        f"{n}:\n{o}" for n, o in survivors)
