"""The C ABI loads, exports every symbol include/sta.h declares, and rejects
bad arguments on the host (no GPU needed, no kernel launched)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_local_attention_b200 import sta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sta.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sta_[a-z_]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(sta.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(sta.library_path())
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    for code in range(9):
        assert sta.status_string(code)
    assert sta.status_string(99) == "unknown status"


def _create(**kw):
    base = dict(batch=1, heads=1, head_dim=64, T=4, H=8, W=8, tile=(2, 4, 4), windows=[(1, 1, 1)], host_only=True)
    base.update(kw)
    return sta.sta_plan_create(sta.Problem(**base))


@pytest.mark.parametrize("kw,code", [
    (dict(T=5), 2),                      # tile does not divide T
    (dict(tile=(3, 4, 4), T=6), 3),      # tile volume 48 ok? 48 % 8 == 0 -> fine below
    (dict(head_dim=96), 3),
    (dict(windows=[(0, 1, 1)]), 1),
    (dict(batch=0), 2),
    (dict(tile=(1, 1, 3), T=4, H=8, W=9), 3),  # tile volume 3, not a multiple of 8
])
def test_plan_rejects_bad_problems(kw, code):
    if kw.get("tile") == (3, 4, 4):
        _create(**kw)  # volume 48 is accepted
        return
    with pytest.raises(sta.StaError) as e:
        _create(**kw)
    assert e.value.status == code


def test_compute_calls_on_host_only_plan_fail_cleanly():
    plan = _create()
    st = sta.lib().sta_forward(plan.handle, None, None, None, None, None, None, 0, None, 0)
    assert st == 1
    st = sta.lib().sta_permute(plan.handle, None, None, 0, None)
    assert st == 1


def test_backward_requires_backward_tables():
    plan = _create()
    with pytest.raises(sta.StaError):
        sta.sta_plan_q_tiles(plan, 0)


@pytest.mark.parametrize("tile,T,H,W,win,forward", [
    ((4, 8, 8), 8, 16, 16, (3, 3, 3), 1),   # 256 tokens: two query blocks per tile
    ((6, 8, 8), 12, 16, 16, (3, 3, 3), 1),  # 384 tokens, one window for all tiles: last blocks pair up
    ((6, 8, 8), 6, 8, 24, (1, 1, 1), 2),    # 384 tokens, every window distinct: lone last blocks
    ((2, 4, 4), 4, 8, 8, (3, 3, 3), 1),     # 32 tokens: one block per tile, paired across tiles
    ((2, 6, 4), 4, 12, 8, (3, 3, 3), 4),    # 48 tokens, not a box of the raster tensor: 3 gathers + pairs
])
def test_plan_launch_counts(tile, T, H, W, win, forward):
    plan = _create(head_dim=128, T=T, H=H, W=W, tile=tile, windows=[win], backward=True)
    assert plan.forward_launches == forward
    gather = forward == 4
    assert plan.backward_launches == (4 if gather else 0) + 3
    plan_f = _create(head_dim=128, T=T, H=H, W=W, tile=tile, windows=[win])
    assert plan_f.backward_launches == 0


def test_plan_rejects_more_rows_than_32_bit_indexing():
    """batch * heads * T*H*W rows index the kernels' 32-bit row space; a
    problem at 2^31 rows is refused before any table is built."""
    with pytest.raises(sta.StaError) as e:
        _create(batch=32, heads=1, T=64, H=1024, W=1024, tile=(1, 8, 8), windows=[(1, 1, 1)])
    assert e.value.status == 2


def test_plan_rejects_lists_past_32_bit_positions():
    """heads * tiles * window tiles list entries are 32-bit positions on the
    device: a plan whose lists reach 2^31 entries is refused before they are
    built, even though its row count fits."""
    # 1 x 1 x 376832 tokens in tiles of 8: 47104 tiles, a window over all of
    # them gives 47104^2 = 2.2e9 list entries
    with pytest.raises(sta.StaError) as e:
        _create(batch=1, heads=1, T=1, H=1, W=376832, tile=(1, 1, 8), windows=[(1, 1, 47104)])
    assert e.value.status == 2
    # the same latent with a window of 64 tiles (3M entries) is planned
    plan = _create(batch=1, heads=1, T=1, H=1, W=376832, tile=(1, 1, 8), windows=[(1, 1, 64)])
    assert plan.n_tiles == 47104


def test_binding_refuses_buffers_the_kernels_cannot_use():
    """The library sees only pointers, so the binding checks every tensor it
    passes (shape, dtype, contiguity, CUDA residency) before any call: host
    tensors, wrong shapes and non-tensors are refused without reaching it."""
    plan = _create(backward=True)
    shape = (1, 1, 4 * 8 * 8, 64)
    x = torch.zeros(shape, dtype=torch.bfloat16)
    lse = torch.zeros(shape[:3], dtype=torch.float32)
    with pytest.raises(ValueError, match="q: expected contiguous"):
        sta.sta_forward(plan, x, x, x)
    with pytest.raises(ValueError, match="src: expected contiguous"):
        sta.sta_permute(plan, x)
    with pytest.raises(ValueError, match="q: expected contiguous"):
        sta.sta_backward(plan, x, x, x, x, lse, x)
    with pytest.raises(ValueError, match="expected contiguous"):
        sta.sta_forward(plan, x[..., :32], x, x)          # wrong head dim
    with pytest.raises(ValueError, match="expected contiguous"):
        sta.sta_forward(plan, x.transpose(2, 3).contiguous().transpose(2, 3), x, x)  # strided
    with pytest.raises(TypeError):
        sta.sta_forward(plan, [0.0] * 64, x, x)
    # host tensors of the right shape are what sta_forward_host takes; its
    # device workspace is checked too
    with pytest.raises(ValueError, match="workspace"):
        sta.sta_forward_host(plan, x, x, x, workspace=torch.zeros(16, dtype=torch.uint8))


class _OnCuda0(torch.Tensor):
    """A host tensor that reports itself as living on cuda:0 (to exercise the
    binding's marshalling of device calls without a GPU)."""

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", 0)


class _OnCuda1(_OnCuda0):
    @property
    def device(self):
        return torch.device("cuda", 1)


class _RecordingLib:
    """Stands in for libsta.so: records each call's arguments, returns STA_OK;
    `devices` records the device current (under _FakeDevices) at each call."""

    def __init__(self, devices=None):
        self.calls = []
        self.devices = []
        self.current = devices

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            self.devices.append(self.current.now if self.current is not None else None)
            return 0
        return call


class _FakeDevices:
    """Stands in for torch.cuda.device / current_device on a machine without
    a GPU: a device context that only records which device it made current."""

    def __init__(self, start=0):
        self.now = start

    def current_device(self):
        return self.now

    def device(self, index):
        fake = self

        class _Ctx:
            def __enter__(self):
                self.prev, fake.now = fake.now, index

            def __exit__(self, *exc):
                fake.now = self.prev
        return _Ctx()


def test_binding_passes_valid_device_buffers_through(monkeypatch):
    """Valid device-side calls pass the binding's checks and reach the library
    with the tensors' own pointers and the workspace size in bytes; buffers of
    another shape, dtype or device are refused."""
    plan = _create(backward=True)
    plan.device = 0  # as if the tables had been uploaded to cuda:0
    shape = (1, 1, 4 * 8 * 8, 64)
    dev = lambda t: t.as_subclass(_OnCuda0)
    q, k, v, o, do = (dev(torch.zeros(shape, dtype=torch.bfloat16)) for _ in range(5))
    lse = dev(torch.zeros(shape[:3], dtype=torch.float32))
    ws = dev(torch.zeros(100, dtype=torch.float32))  # 400 bytes
    fake = _FakeDevices()
    monkeypatch.setattr(torch.cuda, "device", fake.device)
    rec = _RecordingLib(fake)
    monkeypatch.setattr(sta, "lib", lambda: rec)

    sta.sta_forward(plan, q, k, v, o, lse, ws, stream=0, check=True)
    name, args = rec.calls[-1]
    assert name == "sta_forward"
    assert [a.value for a in args[1:7]] == [t.data_ptr() for t in (q, k, v, o, lse, ws)]
    assert args[7] == 400 and args[9] == sta.STA_CALL_CHECK

    dq, dk, dv = sta.sta_backward(plan, q, k, v, o, lse, do, workspace=ws, stream=0)
    name, args = rec.calls[-1]
    assert name == "sta_backward" and args[11] == 400
    assert [a.value for a in args[7:10]] == [t.data_ptr() for t in (dq, dk, dv)]
    assert all(t.shape == q.shape and t.dtype == torch.bfloat16 for t in (dq, dk, dv))

    dst = sta.sta_permute(plan, q, stream=0, inverse=True)
    name, args = rec.calls[-1]
    assert name == "sta_permute" and args[2].value == dst.data_ptr() and args[3] == 1

    qh = torch.zeros(shape, dtype=torch.bfloat16)
    oh, lh = sta.sta_forward_host(plan, qh, qh, qh, workspace=ws, stream=0)
    name, args = rec.calls[-1]
    assert name == "sta_forward_host" and args[7] == 400
    assert oh.shape == shape and not oh.is_cuda and lh.shape == shape[:3]

    n = len(rec.calls)
    bad = [
        dict(o=dev(torch.zeros(shape[:3] + (32,), dtype=torch.bfloat16))),   # o: wrong head dim
        dict(lse=dev(torch.zeros(shape[:3], dtype=torch.bfloat16))),         # lse: wrong dtype
        dict(o=torch.zeros(shape, dtype=torch.bfloat16).as_subclass(_OnCuda1)),  # o: another GPU
        dict(workspace=torch.zeros(400, dtype=torch.uint8)),                  # host workspace
    ]
    for kw in bad:
        args = dict(o=o, lse=lse, workspace=ws)
        args.update(kw)
        with pytest.raises(ValueError):
            sta.sta_forward(plan, q, k, v, stream=0, **args)
    with pytest.raises(ValueError, match="dk"):
        sta.sta_backward(plan, q, k, v, o, lse, do, dk=dev(torch.zeros(shape, dtype=torch.float32)),
                         workspace=ws, stream=0)
    assert len(rec.calls) == n  # none of them reached the library
    plan.device = None  # it is a host-only plan again when it is freed


def test_planner_reports_out_of_memory(tmp_path):
    """A host allocation failure inside sta_plan_create (injected by capping
    the process's address space, in a C program of its own) is STA_ERR_OOM,
    leaves the output handle untouched, and the library keeps working."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_oom"
    lib_dir = os.path.dirname(sta.library_path())
    subprocess.run(["gcc", "-std=gnu99", "-O1", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_oom.c"), "-L", lib_dir, "-lsta",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert got == {"big_status": "6", "big_untouched": "1", "small_status": "0"}


def test_c_program_on_the_abi(tmp_path):
    """A plain C program (no Python, no torch) compiled against include/sta.h
    and linked to libsta.so: host-only plan calls give what the binding gives."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_host"
    lib_dir = os.path.dirname(sta.library_path())
    subprocess.run(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_host.c"), "-L", lib_dir, "-lsta",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    plan = _create(head_dim=128, heads=2, T=12, H=16, W=16, tile=(6, 8, 8), windows=[(3, 3, 3), (1, 1, 1)],
                   backward=True)
    kv = sta.sta_plan_kv_tiles(plan, 0)
    assert got["create"] == "0"
    assert int(got["tiles"]) == plan.n_tiles and int(got["tau"]) == plan.tile_volume
    assert int(got["fwd_launches"]) == plan.forward_launches
    assert int(got["bwd_launches"]) == plan.backward_launches
    assert int(got["fwd_bytes"]) == plan.fwd_workspace_bytes and int(got["bwd_bytes"]) == plan.bwd_workspace_bytes
    assert int(got["host_bytes"]) == plan.host_workspace_bytes
    assert int(got["kv_entries_head0"]) == kv.numel()
    assert int(got["kv_tile0_first"]) == int(kv[0, 0]) and int(got["kv_tile0_last"]) == int(kv[0, -1])
    assert got["forward_on_host_plan"] == "1"
    assert got["bad_shape"] == "2" and got["bad_head_dim"] == "3"
    assert got["status_8"] == sta.status_string(8)


def test_autograd_and_plan_cache_marshalling(monkeypatch):
    """sliding_tile_attention: the forward is one sta_forward call, the
    backward one sta_backward call on the saved q, k, v, o, lse with the
    incoming gradient, and its dq, dk, dv are the gradients autograd returns;
    plans come from a bounded cache keyed by the problem.  (Fake cuda:0
    tensors and a recording library: no GPU.)"""
    from collections import OrderedDict
    rec = _RecordingLib()
    monkeypatch.setattr(sta, "lib", lambda: rec)
    monkeypatch.setattr(sta, "_PLANS", OrderedDict())
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "device", _FakeDevices().device)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(sta, "_stream", lambda stream: ctypes.c_void_p(0))

    def expect_shape(t, name, shape, dtype, device=None):
        # autograd hands saved tensors back as plain (host) tensors, so only
        # shape and dtype are checked here; the device checks have their own tests
        assert tuple(t.shape) == tuple(shape) and t.dtype == dtype, name
    monkeypatch.setattr(sta, "_expect", expect_shape)
    monkeypatch.setattr(sta.Plan, "workspace",
                        lambda self, **kw: torch.zeros(256, dtype=torch.uint8).as_subclass(_OnCuda0))
    T, H, W, tile = 4, 8, 8, (2, 4, 4)
    shape = (1, 2, T * H * W, 64)
    q, k, v = (torch.randn(shape).to(torch.bfloat16).as_subclass(_OnCuda0).requires_grad_() for _ in range(3))

    o = sta.sliding_tile_attention(q, k, v, T, H, W, tile, (3, 3, 3))
    assert [c[0] for c in rec.calls].count("sta_plan_create") == 1
    fwd = [c for c in rec.calls if c[0] == "sta_forward"][-1][1]
    assert [a.value for a in fwd[1:4]] == [t.data_ptr() for t in (q, k, v)]
    assert fwd[4].value == o.data_ptr() and fwd[5].value is not None  # LSE kept for the backward

    do = torch.randn(shape).to(torch.bfloat16).as_subclass(_OnCuda0)
    grads = torch.autograd.grad(o, (q, k, v), grad_outputs=do)
    bwd = [c for c in rec.calls if c[0] == "sta_backward"][-1][1]
    assert [a.value for a in bwd[1:5]] == [t.data_ptr() for t in (q, k, v, o)]
    assert bwd[5].value == fwd[5].value and bwd[6].value == do.data_ptr()
    assert [a.value for a in bwd[7:10]] == [g.data_ptr() for g in grads]

    # the same problem reuses its plan; other windows get their own; no grad -> no LSE
    with torch.no_grad():
        sta.sliding_tile_attention(q, k, v, T, H, W, tile, [(3, 3, 3), (3, 3, 3)])
        assert [c[0] for c in rec.calls].count("sta_plan_create") == 1
        assert [c for c in rec.calls if c[0] == "sta_forward"][-1][1][5] is None
        sta.sliding_tile_attention(q, k, v, T, H, W, tile, [(1, 1, 1), (3, 3, 3)])
    assert [c[0] for c in rec.calls].count("sta_plan_create") == 2
    monkeypatch.setattr(sta, "PLAN_CACHE_SIZE", 2)
    with torch.no_grad():
        for w in ((1, 1, 1), (2, 2, 2), (1, 2, 1)):
            sta.sliding_tile_attention(q, k, v, T, H, W, tile, w)
    assert len(sta._PLANS) == 2
    with pytest.raises(ValueError):
        sta.sliding_tile_attention(q, k, v, T, H, W, tile, [(3, 3, 3)] * 3)  # 3 windows, 2 heads


def test_dropped_plans_are_freed_at_the_next_safe_point():
    """A plan the garbage collector drops is not freed inside __del__ (which
    may run during a CUDA-graph capture, where the device cannot be
    synchronised) but queued, and freed by the next plan creation or destroy."""
    import gc
    sta._free_dropped_plans()
    assert sta._DROPPED == []
    plan = _create()
    handle = plan.handle.value
    del plan
    gc.collect()
    assert [h.value for h, _ in sta._DROPPED] == [handle]
    other = _create()                      # a safe point: the dropped plan is freed
    assert sta._DROPPED == []
    other.destroy()
    assert other.handle is None and sta._DROPPED == []


def test_binding_makes_the_plan_device_current_for_each_call(monkeypatch):
    """The library enqueues on the current device and refuses a call made
    while another device is current, so the binding makes the plan's device
    current around every compute call (and only there): a plan of cuda:1 used
    while cuda:0 is current still runs on cuda:1."""
    plan = _create(backward=True)
    plan.device = 1  # as if the tables had been uploaded to cuda:1
    shape = (1, 1, 4 * 8 * 8, 64)
    dev = lambda t: t.as_subclass(_OnCuda1)
    q, o, do = (dev(torch.zeros(shape, dtype=torch.bfloat16)) for _ in range(3))
    lse = dev(torch.zeros(shape[:3], dtype=torch.float32))
    ws = dev(torch.zeros(100, dtype=torch.float32))
    fake = _FakeDevices(start=0)
    monkeypatch.setattr(torch.cuda, "device", fake.device)
    rec = _RecordingLib(fake)
    monkeypatch.setattr(sta, "lib", lambda: rec)
    sta.sta_forward(plan, q, q, q, o, lse, ws, stream=0)
    sta.sta_backward(plan, q, q, q, o, lse, do, q.clone(), q.clone(), q.clone(), workspace=ws, stream=0)
    sta.sta_backward_noalloc(plan, q, q, q, o, lse, do, q.clone(), q.clone(), q.clone(), stream=0)
    sta.sta_permute(plan, q, o, stream=0)
    qh = torch.zeros(shape, dtype=torch.bfloat16)
    sta.sta_forward_host(plan, qh, qh, qh, workspace=ws, stream=0)
    names = [c[0] for c in rec.calls]
    assert names == ["sta_forward", "sta_backward", "sta_backward_noalloc", "sta_permute", "sta_forward_host"]
    assert rec.devices == [1] * 5
    assert fake.now == 0  # the caller's device is current again afterwards
    plan.device = None


def test_noalloc_checks_its_arguments_before_anything_else():
    """sta_backward_noalloc applies sta_backward's argument checks before it
    looks up its scratch array or enqueues anything: a host-only plan is an
    invalid argument (not a CUDA error), as are null tensors and unknown
    flags; misaligned tensors are an alignment error."""
    plan = _create(backward=True)
    L = sta.lib()
    ok = [ctypes.c_void_p(256 * (i + 1)) for i in range(9)]
    assert L.sta_backward_noalloc(plan.handle, *ok, None, 0) == 1           # host-only plan
    fwd_only = _create()
    assert L.sta_backward_noalloc(fwd_only.handle, *ok, None, 0) == 1       # host-only, no backward tables
    assert L.sta_backward_noalloc(None, *ok, None, 0) == 1
