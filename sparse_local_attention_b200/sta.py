"""Python binding of libsta.so (ctypes).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels behind the C ABI of include/sta.h.  PyTorch supplies device memory and
the current stream.  There is no fallback: if the library cannot be loaded the
call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from collections import OrderedDict
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

from . import _build

STA_OK = 0
STATUS_NAMES = {0: "STA_OK", 1: "STA_ERR_INVALID_ARG", 2: "STA_ERR_SHAPE", 3: "STA_ERR_UNSUPPORTED",
                4: "STA_ERR_ALIGNMENT", 5: "STA_ERR_WORKSPACE", 6: "STA_ERR_OOM", 7: "STA_ERR_CUDA",
                8: "STA_ERR_TIMEOUT"}
STA_PROBLEM_BACKWARD = 0x1
STA_PROBLEM_TILED = 0x2
STA_PROBLEM_HOST_ONLY = 0x4
STA_PROBLEM_DEVICE_CHECK_TEST = 0x10
STA_CALL_CHECK = 0x1

EXPORTED = ["sta_plan_create", "sta_plan_destroy", "sta_plan_workspace_size", "sta_plan_kv_tiles",
            "sta_plan_q_tiles", "sta_plan_geometry", "sta_permute", "sta_forward", "sta_backward",
            "sta_status_string", "sta_set_wait_limit_ns", "sta_backward_noalloc", "sta_plan_launches",
            "sta_plan_host_workspace_size", "sta_forward_host", "sta_plan_work_items"]
STA_WORK_FORWARD, STA_WORK_FORWARD_HOST, STA_WORK_DKDV, STA_WORK_DQ = 0, 1, 2, 3


class StaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


class _Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("tile_t", ctypes.c_int32), ("tile_h", ctypes.c_int32), ("tile_w", ctypes.c_int32),
                ("window", ctypes.POINTER(ctypes.c_int32)), ("scale", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


_lib = None


def library_path() -> str:
    """libsta.so as built in-tree, or the build STA_LIBRARY names (the
    planner's mutation tests load copies with a planted mistake that way)."""
    return os.environ.get("STA_LIBRARY") or _build.LIB


def lib() -> ctypes.CDLL:
    """Load libsta.so (building it with nvcc first if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if path == _build.LIB and not os.path.exists(path):
        _build.build()
    L = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    szp = ctypes.POINTER(ctypes.c_size_t)
    i32p = ctypes.POINTER(ctypes.c_int32)
    L.sta_plan_create.argtypes = [ctypes.POINTER(_Problem), ctypes.POINTER(vp)]
    L.sta_plan_destroy.argtypes = [vp]
    L.sta_plan_workspace_size.argtypes = [vp, szp, szp]
    L.sta_plan_kv_tiles.argtypes = [vp, ctypes.c_int32, i32p, sz, szp]
    L.sta_plan_q_tiles.argtypes = [vp, ctypes.c_int32, i32p, i32p, sz, szp]
    L.sta_plan_geometry.argtypes = [vp, i32p, i32p]
    L.sta_permute.argtypes = [vp, vp, vp, ctypes.c_int32, vp]
    L.sta_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.c_uint32]
    L.sta_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.c_uint32]
    L.sta_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_uint32]
    L.sta_plan_launches.argtypes = [vp, i32p, i32p]
    L.sta_plan_host_workspace_size.argtypes = [vp, szp]
    L.sta_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.c_uint32]
    L.sta_plan_work_items.argtypes = [vp, ctypes.c_int32, i32p, sz, szp, i32p]
    L.sta_status_string.argtypes = [ctypes.c_int]
    L.sta_status_string.restype = ctypes.c_char_p
    L.sta_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.sta_set_wait_limit_ns.restype = None
    for name in EXPORTED:
        if name not in ("sta_status_string", "sta_set_wait_limit_ns"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().sta_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != STA_OK:
        raise StaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


@dataclass
class Problem:
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    tile: tuple
    windows: Sequence  # per head (w_t, w_h, w_w)
    scale: float = 0.0
    backward: bool = False
    tiled: bool = False
    host_only: bool = False
    extra_flags: int = 0  # other STA_PROBLEM_* bits (the device-check test flag)

    def _c(self):
        flat = [int(x) for w in self.windows for x in w]
        arr = (ctypes.c_int32 * max(1, len(flat)))(*flat)
        flags = ((STA_PROBLEM_BACKWARD if self.backward else 0) | (STA_PROBLEM_TILED if self.tiled else 0)
                 | (STA_PROBLEM_HOST_ONLY if self.host_only else 0) | int(self.extra_flags))
        p = _Problem(self.batch, self.heads, self.head_dim, self.T, self.H, self.W, *self.tile,
                     ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)), float(self.scale), flags)
        return p, arr

    @staticmethod
    def from_workload(wl, backward=None, tiled=False, host_only=False, scale=0.0) -> "Problem":
        return Problem(wl.B, wl.Hh, wl.d, wl.T, wl.H, wl.W, tuple(wl.tile), tuple(wl.windows), scale,
                       bool(wl.backward if backward is None else backward), tiled, host_only)


# Plans the garbage collector dropped without destroy(): (handle, device).
# They are freed at the next safe point (see _free_dropped_plans).
_DROPPED: list = []


def _capturing() -> bool:
    return torch.cuda.is_available() and torch.cuda.is_current_stream_capturing()


def _free_dropped_plans():
    """Free the plans the garbage collector dropped.  Kernels still queued may
    read their tables, so each plan's device is synchronised first -- which is
    not allowed while a stream is being captured into a CUDA graph, so then
    they wait for the next call."""
    if not _DROPPED or _capturing():
        return
    while _DROPPED:
        handle, device = _DROPPED.pop()
        try:
            if device is not None:
                torch.cuda.synchronize(device)
        finally:
            lib().sta_plan_destroy(handle)


class Plan:
    """Owns an sta_plan_t.  Create with sta_plan_create()."""

    def __init__(self, handle: ctypes.c_void_p, problem: Problem):
        self.handle = handle
        self.problem = problem
        fwd, bwd = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().sta_plan_workspace_size(handle, ctypes.byref(fwd), ctypes.byref(bwd)), "sta_plan_workspace_size")
        self.fwd_workspace_bytes = fwd.value
        self.bwd_workspace_bytes = bwd.value
        nt, tv = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().sta_plan_geometry(handle, ctypes.byref(nt), ctypes.byref(tv)), "sta_plan_geometry")
        self.n_tiles, self.tile_volume = nt.value, tv.value
        fl, bl = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().sta_plan_launches(handle, ctypes.byref(fl), ctypes.byref(bl)), "sta_plan_launches")
        self.forward_launches, self.backward_launches = fl.value, bl.value  # kernels per call
        hb = ctypes.c_size_t()
        _check(lib().sta_plan_host_workspace_size(handle, ctypes.byref(hb)), "sta_plan_host_workspace_size")
        self.host_workspace_bytes = hb.value
        # the device the tables were uploaded to; every tensor of a call must live there
        self.device = None if problem.host_only else torch.cuda.current_device()

    def destroy(self):
        """Free the plan.  Its device tables are read by every launch that uses
        it, so the plan's device is synchronised first: no such launch can
        still be running when they are freed.  Call it outside stream capture."""
        if self.handle is not None and self.handle.value:
            if self.device is not None:
                torch.cuda.synchronize(self.device)
            _check(lib().sta_plan_destroy(self.handle), "sta_plan_destroy")
        self.handle = None
        _free_dropped_plans()

    def __del__(self):
        # The garbage collector runs anywhere -- inside a CUDA-graph capture
        # too, where synchronising the device would break the capture -- so a
        # dropped plan is only queued here and freed at the next safe point.
        try:
            if self.handle is not None and self.handle.value:
                _DROPPED.append((self.handle, self.device))
            self.handle = None
        except Exception:
            pass

    def workspace(self, backward=False, device=None, host=False) -> torch.Tensor:
        """Device workspace for sta_forward, sta_backward (backward=True) or
        sta_forward_host (host=True), on the plan's device."""
        n = self.host_workspace_bytes if host else self.bwd_workspace_bytes if backward else self.fwd_workspace_bytes
        if device is None:
            device = torch.device("cuda", self.device) if self.device is not None else "cuda"
        return torch.empty(n, dtype=torch.uint8, device=device)


def sta_plan_create(problem: Problem) -> Plan:
    _free_dropped_plans()
    cp, keep = problem._c()
    h = ctypes.c_void_p()
    _check(lib().sta_plan_create(ctypes.byref(cp), ctypes.byref(h)), "sta_plan_create")
    del keep
    return Plan(h, problem)


def sta_plan_destroy(plan: Plan):
    plan.destroy()


def sta_plan_workspace_size(plan: Plan):
    return plan.fwd_workspace_bytes, plan.bwd_workspace_bytes


def sta_plan_kv_tiles(plan: Plan, head: int) -> torch.Tensor:
    """[n_tiles, per_tile] int32 KV-tile lists of one head (host copy)."""
    n = ctypes.c_size_t()
    _check(lib().sta_plan_kv_tiles(plan.handle, head, None, 0, ctypes.byref(n)), "sta_plan_kv_tiles")
    out = torch.empty(n.value, dtype=torch.int32)
    _check(lib().sta_plan_kv_tiles(plan.handle, head, ctypes.cast(out.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
                                   n.value, ctypes.byref(n)), "sta_plan_kv_tiles")
    return out.view(plan.n_tiles, -1)


def sta_plan_work_items(plan: Plan, which: int):
    """(items, n_lone): one of the plan's work lists as an int32 [n, 4]
    (forward lists) or [n, 2] (backward lists) host tensor; see include/sta.h."""
    n, lone = ctypes.c_size_t(), ctypes.c_int32()
    _check(lib().sta_plan_work_items(plan.handle, which, None, 0, ctypes.byref(n), ctypes.byref(lone)),
           "sta_plan_work_items")
    width = 4 if which in (STA_WORK_FORWARD, STA_WORK_FORWARD_HOST) else 2
    out = torch.empty(max(1, n.value) * width, dtype=torch.int32)
    _check(lib().sta_plan_work_items(plan.handle, which, ctypes.cast(out.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
                                     n.value, ctypes.byref(n), None), "sta_plan_work_items")
    return out[: n.value * width].view(n.value, width), lone.value


def sta_plan_q_tiles(plan: Plan, head: int):
    """(offsets[n_tiles + 1], indices) inverse lists of one head (host copy)."""
    n = ctypes.c_size_t()
    _check(lib().sta_plan_q_tiles(plan.handle, head, None, None, 0, ctypes.byref(n)), "sta_plan_q_tiles")
    off = torch.empty(plan.n_tiles + 1, dtype=torch.int32)
    idx = torch.empty(max(1, n.value), dtype=torch.int32)
    i32p = ctypes.POINTER(ctypes.c_int32)
    _check(lib().sta_plan_q_tiles(plan.handle, head, ctypes.cast(off.data_ptr(), i32p),
                                  ctypes.cast(idx.data_ptr(), i32p), n.value, ctypes.byref(n)), "sta_plan_q_tiles")
    return off, idx[: n.value]


def _shape(plan: Plan):
    p = plan.problem
    return (p.batch, p.heads, p.T * p.H * p.W, p.head_dim)


def _expect(t: torch.Tensor, name: str, shape, dtype, device: Optional[int] = None):
    """A tensor handed to the kernels: contiguous, on the plan's CUDA device,
    of exactly the shape and dtype the C ABI assumes (the library sees only a
    pointer, so a wrong buffer would be read or written out of bounds)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    on_device = t.is_cuda and (device is None or t.device.index == device)
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not on_device:
        where = f"cuda:{device}" if device is not None else "CUDA"
        raise ValueError(f"{name}: expected contiguous {where} {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()} on {t.device}")


def _workspace(plan: Plan, ws: Optional[torch.Tensor], **kind):
    """The caller's workspace (contiguous device memory on the plan's device;
    its size in bytes goes to the library, which checks it), or a new one."""
    if ws is None:
        return plan.workspace(**kind)
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous() or (
            plan.device is not None and ws.device.index != plan.device):
        raise ValueError("workspace: expected a contiguous tensor on the plan's CUDA device")
    return ws


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _on_plan_device(plan: Plan):
    """Context in which a compute call runs: the plan's device made current.
    The library enqueues on the current device (and refuses a call made while
    another device is current), and the default stream of a call is the
    current stream of that device."""
    if plan.device is None:
        return contextlib.nullcontext()
    return torch.cuda.device(plan.device)


def sta_permute(plan: Plan, src: torch.Tensor, dst: Optional[torch.Tensor] = None, inverse: bool = False,
                stream=None) -> torch.Tensor:
    _expect(src, "src", _shape(plan), torch.bfloat16, plan.device)
    if dst is None:
        dst = torch.empty_like(src)
    _expect(dst, "dst", _shape(plan), torch.bfloat16, plan.device)
    with _on_plan_device(plan):
        _check(lib().sta_permute(plan.handle, _ptr(src), _ptr(dst), 1 if inverse else 0, _stream(stream)),
               "sta_permute")
    return dst


def sta_forward(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                check: bool = False, want_lse: bool = True):
    shape, dev = _shape(plan), plan.device
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _expect(t, nm, shape, torch.bfloat16, dev)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = q.new_empty(shape[:3], dtype=torch.float32)
    _expect(o, "o", shape, torch.bfloat16, dev)
    if lse is not None:
        _expect(lse, "lse", shape[:3], torch.float32, dev)
    workspace = _workspace(plan, workspace)
    with _on_plan_device(plan):
        st = lib().sta_forward(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace),
                               _nbytes(workspace), _stream(stream), STA_CALL_CHECK if check else 0)
    _check(st, "sta_forward")
    return o, lse


def _expect_host(t: torch.Tensor, name: str, shape, dtype):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or t.is_cuda:
        raise ValueError(f"{name}: expected contiguous host {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()} cuda={t.is_cuda}")


def sta_forward_host(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                     check: bool = False, want_lse: bool = True):
    """Forward pass on host tensors (pin them for the copies to overlap the
    kernels); returns host (o, lse).  The outputs are complete once `stream`
    (default: the current stream) has passed the call."""
    shape = _shape(plan)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _expect_host(t, nm, shape, torch.bfloat16)
    if o is None:
        o = torch.empty(shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    if lse is None and want_lse:
        lse = torch.empty(shape[:3], dtype=torch.float32, pin_memory=q.is_pinned())
    _expect_host(o, "o", shape, torch.bfloat16)
    if lse is not None:
        _expect_host(lse, "lse", shape[:3], torch.float32)
    workspace = _workspace(plan, workspace, host=True)
    with _on_plan_device(plan):
        st = lib().sta_forward_host(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace),
                                    _nbytes(workspace), _stream(stream), STA_CALL_CHECK if check else 0)
    _check(st, "sta_forward_host")
    return o, lse


def sta_backward(plan: Plan, q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, stream=None,
                 check: bool = False):
    shape, dev = _shape(plan), plan.device
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _expect(t, nm, shape, torch.bfloat16, dev)
    _expect(lse, "lse", shape[:3], torch.float32, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, nm in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _expect(t, nm, shape, torch.bfloat16, dev)
    workspace = _workspace(plan, workspace, backward=True)
    with _on_plan_device(plan):
        st = lib().sta_backward(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace), _stream(stream),
                                STA_CALL_CHECK if check else 0)
    _check(st, "sta_backward")
    return dq, dk, dv


def sta_backward_noalloc(plan: Plan, q, k, v, o, lse, dout, dq=None, dk=None, dv=None, stream=None,
                         check: bool = False):
    """sta_backward with the library's fixed device scratch instead of a
    workspace (see include/sta.h).  Output tensors may be passed in; if they
    are not, they are created here by the caller's allocator (torch)."""
    shape, dev = _shape(plan), plan.device
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _expect(t, nm, shape, torch.bfloat16, dev)
    _expect(lse, "lse", shape[:3], torch.float32, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, nm in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _expect(t, nm, shape, torch.bfloat16, dev)
    with _on_plan_device(plan):
        st = lib().sta_backward_noalloc(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                        _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream), STA_CALL_CHECK if check else 0)
    _check(st, "sta_backward_noalloc")
    return dq, dk, dv


def sta_set_wait_limit_ns(ns: int):
    lib().sta_set_wait_limit_ns(int(ns))


class _SlidingTileAttention(torch.autograd.Function):
    """O = STA(q, k, v) with its gradient: sta_forward saves LSE, and the
    backward is one sta_backward call (the plan must carry the inverse lists)."""

    @staticmethod
    def forward(ctx, q, k, v, plan):
        o, lse = sta_forward(plan, q, k, v)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.plan = plan
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = sta_backward(ctx.plan, q, k, v, o, lse, do.contiguous())
        return dq, dk, dv, None


_PLANS: "OrderedDict[tuple, Plan]" = OrderedDict()
_PLANS_LOCK = threading.Lock()
PLAN_CACHE_SIZE = 16


def cached_plan(problem: Problem) -> Plan:
    """The plan of `problem` on the current device, built on first use and
    kept (the PLAN_CACHE_SIZE most recently used).  A plan that leaves the
    cache is freed once nothing refers to it any more (an autograd graph may
    still hold it for its backward)."""
    key = (problem.batch, problem.heads, problem.head_dim, problem.T, problem.H, problem.W, tuple(problem.tile),
           tuple(tuple(int(x) for x in w) for w in problem.windows), float(problem.scale), problem.backward,
           problem.tiled, problem.extra_flags, torch.cuda.current_device())
    with _PLANS_LOCK:
        plan = _PLANS.get(key)
        if plan is not None:
            _PLANS.move_to_end(key)
            return plan
        plan = sta_plan_create(problem)
        _PLANS[key] = plan
        while len(_PLANS) > PLAN_CACHE_SIZE:
            _PLANS.popitem(last=False)
        return plan


def _per_head(windows, heads: int):
    """One (w_t, w_h, w_w) for every head, or one per head."""
    if len(windows) == 3 and all(isinstance(x, int) for x in windows):
        return tuple([tuple(int(x) for x in windows)] * heads)
    if len(windows) != heads:
        raise ValueError(f"{len(windows)} windows for {heads} heads")
    return tuple(tuple(int(x) for x in w) for w in windows)


def sliding_tile_attention(q, k, v, T, H, W, tile, windows, scale=0.0):
    """Sliding Tile Attention of bf16 [batch, heads, T*H*W, d] tensors in
    raster token order; returns O (same shape).  `windows`: one (w_t, w_h, w_w)
    in tiles for every head, or one per head.  Differentiable: when q, k or v
    requires a gradient, the backward runs sta_backward.  The plan comes from
    a small cache keyed by the problem, so repeated calls do not rebuild it.
    Non-contiguous inputs are made contiguous first."""
    B, Hh, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"token count {N} != T*H*W = {T * H * W}")
    plan = cached_plan(Problem(B, Hh, d, T, H, W, tuple(tile), _per_head(windows, Hh), scale, backward=True))
    q, k, v = (t.contiguous() for t in (q, k, v))
    if torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v)):
        return _SlidingTileAttention.apply(q, k, v, plan)
    o, _ = sta_forward(plan, q, k, v, want_lse=False)
    return o
