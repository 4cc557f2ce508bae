"""fp64 CPU oracle for Sliding Tile Attention (STA).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA product path (``sparse_local_attention_b200``) never imports
it, and the two share no code: this package wraps ``sta_oracle.c`` only.

What the oracle computes is the plain definition of STA ("Fast Video Generation
with Sliding Tile Attention", Abstract; summary page, Methodology and Novelty):
for every query token, the keys of the whole tiles inside the query tile's 3D
window, softmax(q.k * scale) over exactly those keys, and the weighted sum of
their values -- in fp64, from explicit per-query membership computed from raw
token coordinates.  The border rule (window centred on the query tile, shifted
inward so it stays inside the grid) is the reading documented in the C file.

Parity status: pinned by ``tests/test_oracle.py`` (no function is unpinned).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sta_oracle.c")
# STA_ORACLE_LIB names a prebuilt oracle library to load instead (the
# mutation tests point it at copies of sta_oracle.c with a planted mistake)
_LIB = os.environ.get("STA_ORACLE_LIB") or os.path.join(_HERE, "libsta_oracle.so")

_lib = None


def compile_command(src: str, out: str) -> list:
    """gcc command that builds the oracle library `out` from `src`."""
    return ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", out, src, "-lm"]


def build(force: bool = False) -> str:
    """Compile sta_oracle.c into libsta_oracle.so (gcc, OpenMP, -O2)."""
    if os.environ.get("STA_ORACLE_LIB"):
        return _LIB
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = compile_command(_SRC, _LIB)
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u16p = ctypes.c_void_p
        f64p = ctypes.c_void_p
        lib.sta_oracle_forward.argtypes = [i32p, i32p, ctypes.c_double, u16p, u16p, u16p,
                                           ctypes.c_long, ctypes.c_void_p, ctypes.c_int,
                                           f64p, f64p]
        lib.sta_oracle_forward.restype = ctypes.c_int
        lib.sta_oracle_probs.argtypes = [i32p, i32p, ctypes.c_double, u16p, u16p, u16p,
                                         ctypes.c_int64, f64p]
        lib.sta_oracle_probs.restype = ctypes.c_int
        lib.sta_oracle_mask.argtypes = [i32p, i32p, ctypes.c_int, ctypes.c_void_p]
        lib.sta_oracle_mask.restype = ctypes.c_int
        lib.sta_oracle_backward.argtypes = [i32p, i32p, ctypes.c_double, u16p, u16p, u16p, u16p,
                                            ctypes.c_int64, ctypes.c_long, ctypes.c_void_p,
                                            ctypes.c_long, ctypes.c_void_p, f64p, f64p, f64p]
        lib.sta_oracle_backward.restype = ctypes.c_int
        lib.sta_oracle_threads.argtypes = []
        lib.sta_oracle_threads.restype = ctypes.c_int
        lib.sta_oracle_set_threads.argtypes = [ctypes.c_int]
        lib.sta_oracle_set_threads.restype = None
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Geometry:
    """Problem geometry in the oracle's own terms (tokens, tiles, heads)."""
    B: int
    Hh: int
    d: int
    T: int
    H: int
    W: int
    tile: tuple  # (tile_t, tile_h, tile_w)
    windows: tuple  # per head (w_t, w_h, w_w), in tiles

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    def dims(self):
        return (ctypes.c_int32 * 9)(self.B, self.Hh, self.d, self.T, self.H, self.W, *self.tile)

    def win(self):
        flat = [int(x) for w in self.windows for x in w]
        assert len(flat) == 3 * self.Hh
        return (ctypes.c_int32 * len(flat))(*flat)


def _u16(t) -> np.ndarray:
    """Raw bf16 bits of a torch bf16 tensor (or a uint16 numpy array)."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _scale(geom: Geometry, scale):
    return float(scale) if scale is not None and scale > 0 else 1.0 / float(np.sqrt(geom.d))


def threads() -> int:
    return int(_load().sta_oracle_threads())


def set_threads(n: int) -> None:
    """Threads for later calls (timing only: every result is independent of it)."""
    _load().sta_oracle_set_threads(int(n))


def forward(geom: Geometry, q, k, v, rows=None, scale=None, exhaustive=False):
    """O (fp64, [len(rows), d]) and LSE (fp64, [len(rows)]) for the given rows.

    q, k, v: bf16 [B, Hh, N, d] (raster token order).  rows: flat indices
    bh*N + n (default: every row)."""
    lib = _load()
    qa, ka, va = _u16(q), _u16(k), _u16(v)
    total = geom.B * geom.Hh * geom.N
    if rows is None:
        rows = np.arange(total, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((len(rows), geom.d), dtype=np.float64)
    lse = np.zeros(len(rows), dtype=np.float64)
    rc = lib.sta_oracle_forward(geom.dims(), geom.win(), _scale(geom, scale),
                                qa.ctypes.data, ka.ctypes.data, va.ctypes.data,
                                len(rows), rows.ctypes.data, 1 if exhaustive else 0,
                                o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"sta_oracle_forward failed ({rc})")
    return o, lse


def probs(geom: Geometry, q, k, v, row: int, scale=None) -> np.ndarray:
    """Attention probabilities of one flat query row over all N keys."""
    lib = _load()
    qa, ka, va = _u16(q), _u16(k), _u16(v)
    p = np.zeros(geom.N, dtype=np.float64)
    rc = lib.sta_oracle_probs(geom.dims(), geom.win(), _scale(geom, scale),
                              qa.ctypes.data, ka.ctypes.data, va.ctypes.data, int(row), p.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"sta_oracle_probs failed ({rc})")
    return p


def mask(geom: Geometry, head: int) -> np.ndarray:
    """Boolean [N, N] membership matrix of one head (query rows, key columns)."""
    lib = _load()
    m = np.zeros((geom.N, geom.N), dtype=np.uint8)
    rc = lib.sta_oracle_mask(geom.dims(), geom.win(), int(head), m.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"sta_oracle_mask failed ({rc})")
    return m.astype(bool)


def backward(geom: Geometry, q, k, v, dout, bh: int, q_rows=None, k_rows=None, scale=None):
    """dQ rows, dK rows, dV rows (fp64) for one (batch*heads) slice bh.

    q_rows / k_rows are token indices 0..N-1 inside that slice."""
    lib = _load()
    qa, ka, va, da = _u16(q), _u16(k), _u16(v), _u16(dout)
    q_rows = np.ascontiguousarray(np.arange(geom.N) if q_rows is None else q_rows, dtype=np.int64)
    k_rows = np.ascontiguousarray(np.arange(geom.N) if k_rows is None else k_rows, dtype=np.int64)
    dq = np.zeros((len(q_rows), geom.d))
    dk = np.zeros((len(k_rows), geom.d))
    dv = np.zeros((len(k_rows), geom.d))
    rc = lib.sta_oracle_backward(geom.dims(), geom.win(), _scale(geom, scale),
                                 qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
                                 int(bh), len(q_rows), q_rows.ctypes.data, len(k_rows),
                                 k_rows.ctypes.data, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"sta_oracle_backward failed ({rc})")
    return dq, dk, dv
