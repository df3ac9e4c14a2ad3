"""CPU-side checks of the C ABI library: it loads, exports every declared
symbol, and its host logic (index map, FLOP count, argument validation) agrees
with the oracle.  No kernel is launched here.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import shifted_window_attention_swattn_b200 as sw
from shifted_window_attention_swattn_b200 import build as sw_build
from shifted_window_attention_swattn_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
I3 = ctypes.c_int * 3


@pytest.fixture(scope="module")
def lib():
    sw_build.build()
    return sw._load()


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(basa_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("basa_swattn_fwd", "basa_swattn_index_map", "basa_swattn_flops",
                 "basa_swattn_last_device_error", "basa_strerror"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a():
    cmd = " ".join(sw_build.command("x.so"))
    assert "arch=compute_100a,code=sm_100a" in cmd


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_host_index_map_equals_oracle_on_workloads(lib, wl):
    for shift in wl.shifts:
        got = sw.index_map_host(wl.grid, wl.win, shift)
        ref, _ = oracle.index_map(*wl.grid, wl.win, shift)
        assert np.array_equal(got, ref), shift


@pytest.mark.parametrize("grid,win,shift", [
    ((1, 4, 4), (1, 2, 2), (0, 1, 1)),
    ((3, 1, 5), (2, 1, 2), (1, 0, 2)),
    ((5, 9, 11), (2, 4, 5), (1, 7, -3)),
    ((1, 20, 28), (1, 7, 9), (0, 3, 5)),
    ((2, 16, 20), (2, 16, 10), (1, 8, 5)),
    ((4, 6, 6), (4, 6, 6), (3, -2, 100)),
    ((7, 3, 2), (1, 1, 1), (6, 2, 1)),
])
def test_host_index_map_equals_oracle(lib, grid, win, shift):
    got = sw.index_map_host(grid, win, shift)
    ref, _ = oracle.index_map(*grid, win, shift)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_flops_equal_oracle(lib, wl):
    assert sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.win) == oracle.flops(
        wl.B, wl.heads, *wl.grid, wl.d, wl.win)
    full = sw.flops(wl.B, wl.heads, wl.grid, wl.d, wl.grid)
    assert full == 4.0 * wl.N * wl.N * wl.d * wl.heads * wl.B


def test_flops_truncated_windows(lib):
    for grid, win in [((3, 5, 7), (2, 2, 3)), ((1, 20, 28), (1, 7, 9))]:
        assert sw.flops(2, 3, grid, 64, win) == oracle.flops(2, 3, *grid, 64, win)


def _fwd(lib, q=16, k=32, v=48, out=4096, B=1, heads=1, grid=(1, 4, 4), d=64,
         win=(1, 2, 2), shift=(0, 0, 0), scale=0.125):
    # Fake, never-dereferenced device addresses: every case below must be
    # rejected by host-side validation before anything touches the GPU.
    return lib.basa_swattn_fwd(ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v),
                               ctypes.c_void_p(out), B, heads, *grid, d, I3(*win), I3(*shift),
                               ctypes.c_float(scale), None)


def test_argument_errors_are_caught_on_the_host(lib):
    big = 1 << 30
    assert _fwd(lib, q=0) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, out=0) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, B=0, out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, heads=-1, out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, grid=(1, 0, 4), out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, win=(1, 5, 2), out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, win=(0, 2, 2), out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan"), out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf"), out=big) == sw.BASA_ERR_INVALID_ARG
    assert _fwd(lib, scale=-0.5, out=big) == sw.BASA_ERR_UNSUPPORTED
    assert _fwd(lib, d=96, out=big) == sw.BASA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256, out=big) == sw.BASA_ERR_UNSUPPORTED
    assert _fwd(lib, grid=(1, 1 << 16, 1 << 16), win=(1, 1, 1), out=big) == sw.BASA_ERR_UNSUPPORTED
    assert _fwd(lib, q=24, out=big) == sw.BASA_ERR_ALIGNMENT
    assert _fwd(lib, out=big + 8) == sw.BASA_ERR_ALIGNMENT
    # out overlapping an input (4x4 grid, d=64: 2 KB per tensor)
    assert _fwd(lib, q=big, k=2 * big, v=3 * big, out=big + 1024) == sw.BASA_ERR_ALIAS


def test_strerror_covers_every_code(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert sw.strerror(code) != "unknown error"
    assert sw.strerror(12345) == "unknown error"


def test_python_binding_rejects_non_cuda_tensors(lib):
    import torch
    q = torch.zeros(1, 16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sw.swattn_fwd(q, q, q, (1, 4, 4), (1, 2, 2), (0, 0, 0))


def test_python_binding_device_check_rejects_host_tensors():
    # the check every entry point applies to its outputs, routes, workspace and
    # extra segment: CUDA tensors on the first input's device, nothing else
    import torch
    dev = torch.device("cuda", 0)
    cpu_out = torch.empty(1, 16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sw._require_on(dev, (("out", cpu_out),))
    with pytest.raises(ValueError):
        sw._require_on(dev, (("routed", torch.zeros(1, 1, 4, dtype=torch.int32)),))
    with pytest.raises(ValueError):
        sw._require_on(dev, (("workspace", None),))
    sw._require_on(dev, ())


def test_shift_schedule_equals_oracle(lib):
    for L in (1, 2, 3, 5, 8, 19, 57):
        for win in ((1, 16, 16), (7, 15, 16), (7, 10, 13), (21, 1, 32), (3, 4, 300)):
            for off in ((0, 0, 0), (1, 5, -3), (-8, 40, 7)):
                assert sw.shift_schedule(L, win, off) == oracle.shift_schedule(L, win, off), (L, win, off)


def test_shift_schedule_argument_errors(lib):
    out = (ctypes.c_int * 30)()
    z = I3(0, 0, 0)
    assert lib.basa_shift_schedule(0, I3(1, 8, 8), z, ctypes.cast(out, ctypes.c_void_p)) == sw.BASA_ERR_INVALID_ARG
    assert lib.basa_shift_schedule(4, I3(1, 0, 8), z, ctypes.cast(out, ctypes.c_void_p)) == sw.BASA_ERR_INVALID_ARG
    assert lib.basa_shift_schedule(4, I3(1, 8, 8), z, None) == sw.BASA_ERR_INVALID_ARG
    with pytest.raises(sw.SwattnError):
        sw.shift_schedule(0, (1, 8, 8))


def test_kv_pool_tokens_equal_oracle(lib):
    for grid in ((1, 64, 64), (21, 60, 104), (3, 10, 13), (2, 5, 7)):
        for pool in ((1, 4, 4), (1, 2, 3), (2, 4, 4), (3, 10, 13), (1, 1, 1)):
            assert sw.kv_pool_tokens(grid, pool) == oracle.n_pooled(*grid, pool)


def test_memory_entry_points_reject_bad_arguments_on_the_host(lib):
    vp = ctypes.c_void_p
    a = vp(1 << 20)          # never dereferenced: every call below fails validation first
    win, shift, pool = I3(1, 4, 4), I3(0, 0, 0), I3(1, 2, 2)
    E = sw.BASA_ERR_INVALID_ARG
    # forward with memory
    assert lib.basa_swattn_fwd_mem(a, a, a, None, None, 8, vp(1 << 24), 1, 1, 1, 8, 8, 128, win, shift, 0.1, None) == E
    assert lib.basa_swattn_fwd_mem(a, a, a, a, a, -1, vp(1 << 24), 1, 1, 1, 8, 8, 128, win, shift, 0.1, None) == E
    assert lib.basa_swattn_fwd_mem(a, a, a, vp((1 << 20) + 8), a, 4, vp(1 << 24), 1, 1, 1, 8, 8, 128, win, shift,
                                   0.1, None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_swattn_fwd_mem(a, a, a, vp(1 << 24), a, 4, vp(1 << 24), 1, 1, 1, 8, 8, 128, win, shift,
                                   0.1, None) == sw.BASA_ERR_ALIAS
    assert lib.basa_swattn_fwd_mem(a, a, a, a, a, 4, vp(1 << 24), 1, 1, 1, 8, 8, 96, win, shift, 0.1,
                                   None) == sw.BASA_ERR_UNSUPPORTED
    # pooling
    assert lib.basa_kv_pool(a, a, None, a, 1, 1, 1, 8, 8, 128, pool, None) == E
    assert lib.basa_kv_pool(a, a, vp(1 << 24), vp(1 << 25), 1, 1, 1, 8, 8, 128, I3(1, 0, 2), None) == E
    assert lib.basa_kv_pool(a, a, vp(1 << 24), vp(1 << 25), 1, 1, 1, 8, 8, 96, pool, None) == sw.BASA_ERR_UNSUPPORTED
    assert lib.basa_kv_pool(a, a, vp((1 << 24) + 4), vp(1 << 25), 1, 1, 1, 8, 8, 128, pool,
                            None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_kv_pool(a, a, a, vp(1 << 25), 1, 1, 1, 8, 8, 128, pool, None) == sw.BASA_ERR_ALIAS


def test_route_workspace_bytes(lib):
    n = ctypes.c_size_t(0)
    assert lib.basa_route_workspace_bytes(2, 3, 4, 9, 10, 64, I3(2, 3, 4), ctypes.byref(n)) == sw.BASA_OK
    assert n.value == 2 * 2 * 3 * oracle.n_windows(4, 9, 10, (2, 3, 4)) * 64 * 4
    assert sw.route_workspace_bytes(1, 40, (21, 45, 80), 128, (7, 15, 16)) == 2 * 40 * 45 * 128 * 4
    assert sw.n_windows((21, 45, 80), (7, 15, 16)) == oracle.n_windows(21, 45, 80, (7, 15, 16))
    assert lib.basa_route_workspace_bytes(1, 1, 1, 8, 8, 96, I3(1, 4, 4), ctypes.byref(n)) == sw.BASA_ERR_UNSUPPORTED


def test_routing_entry_points_reject_bad_arguments_on_the_host(lib):
    vp = ctypes.c_void_p
    a = vp(1 << 20)          # never dereferenced: every call below fails validation first
    ws, rt = vp(1 << 24), vp(1 << 25)
    win, shift = I3(1, 4, 4), I3(0, 0, 0)
    E = sw.BASA_ERR_INVALID_ARG
    need = 2 * 4 * 128 * 4   # 1 x 1 x 4 windows x d 128, two fp32 arrays
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, None, need, rt, None) == E
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, ws, need, None, None) == E
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, -1, ws, need, rt, None) == E
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, ws, need - 1, rt, None) == E
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, I3(1, 9, 4), shift, 1, ws, need, rt, None) == E
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 96, win, shift, 1, ws, need, rt, None) == sw.BASA_ERR_UNSUPPORTED
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, vp((1 << 24) + 8), need, rt,
                          None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, ws, need, vp((1 << 25) + 2),
                          None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, ws, need, vp((1 << 20) + 64),
                          None) == sw.BASA_ERR_ALIAS
    assert lib.basa_route(a, a, 1, 1, 1, 8, 8, 128, win, shift, 1, ws, need, vp((1 << 24) + 64),
                          None) == sw.BASA_ERR_ALIAS
    # the routed forward
    out = vp(1 << 26)
    assert lib.basa_swattn_fwd_route(a, a, a, None, None, None, 0, out, 1, 1, 1, 8, 8, 128, win, shift, 0.1,
                                     None) == E
    assert lib.basa_swattn_fwd_route(a, a, a, rt, None, None, 4, out, 1, 1, 1, 8, 8, 128, win, shift, 0.1,
                                     None) == E
    assert lib.basa_swattn_fwd_route(a, a, a, vp((1 << 25) + 2), None, None, 0, out, 1, 1, 1, 8, 8, 128, win,
                                     shift, 0.1, None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_swattn_fwd_route(a, a, a, vp((1 << 26) + 64), None, None, 0, out, 1, 1, 1, 8, 8, 128, win,
                                     shift, 0.1, None) == sw.BASA_ERR_ALIAS
    assert lib.basa_swattn_fwd_route(a, a, a, rt, None, None, 0, out, 1, 1, 1, 8, 8, 96, win, shift, 0.1,
                                     None) == sw.BASA_ERR_UNSUPPORTED


def test_python_binding_routing_rejects_bad_tensors(lib):
    import torch
    q = torch.zeros(1, 16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sw.route(q, q, (1, 4, 4), (1, 2, 2), (0, 0, 0))
    with pytest.raises(TypeError):
        sw.route(q.float(), q.float(), (1, 4, 4), (1, 2, 2), (0, 0, 0))
    routed = torch.zeros(1, 1, 4, dtype=torch.int32)
    with pytest.raises((TypeError, ValueError)):
        sw.swattn_fwd_route(q, q, q, routed, (1, 4, 4), (1, 2, 2), (0, 0, 0))
    with pytest.raises(ValueError):
        sw.n_windows((1, 4, 4), (1, 0, 2))
    assert sw.n_windows((3, 10, 13), (2, 4, 5)) == oracle.n_windows(3, 10, 13, (2, 4, 5))
