"""basa_route_noalloc: top-1 true-window routing for callers that cannot
allocate device memory when they route (code inside another framework's
execution step, such as a plugin's enqueue callback or a serving loop with a
fixed memory budget, where cudaMalloc is forbidden or would stall the device).

The entry point keeps its window descriptors in a fixed array inside the
library instead of a caller's workspace.  Its routes must equal those of
basa_route, the entry point that takes a workspace, exactly (they are integer
window indices computed by the same kernels in the same fixed order), call
after call: the array keeps whatever the previous call left in it.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import shifted_window_attention_swattn_b200 as sw
from shifted_window_attention_swattn_b200.inputs import BY_NAME, make_custom, make_qkv

I3 = ctypes.c_int * 3


def _noalloc(q, k, grid, win, shift, radius, out):
    """One call of the C entry point, with q's device current and its current stream."""
    lib = sw._load()
    B, _, heads, d = q.shape
    vp = ctypes.c_void_p
    with torch.cuda.device(q.device):
        stream = vp(torch.cuda.current_stream(q.device).cuda_stream)
        return lib.basa_route_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), B, heads, *grid, d, I3(*win),
                                      I3(*shift), int(radius), vp(out.data_ptr()), stream)


# (B, heads, d, grid, win, shift, radius, seed): two different problems, so the
# second call finds the first one's descriptors in the shared array
CASES = [
    (1, 4, 128, (3, 20, 26), (3, 5, 6), (0, 2, 3), 1, 31),
    (2, 3, 64, (4, 17, 22), (2, 6, 5), (1, 3, 2), 2, 32),
]


@pytest.mark.gpu
def test_noalloc_routes_equal_workspace_routes_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    for B, heads, d, grid, win, shift, radius, seed in CASES:
        q, k, _ = make_custom(B, heads, d, *grid, seed=seed)
        qd, kd = q.to(dev), k.to(dev)
        out = torch.full((B, heads, sw.n_windows(grid, win)), -7, dtype=torch.int32, device=dev)
        rc = _noalloc(qd, kd, grid, win, shift, radius, out)
        assert rc == sw.BASA_OK, sw.strerror(rc)
        ref = sw.route(qd, kd, grid, win, shift, radius)
        torch.cuda.synchronize()
        assert sw.last_device_error() == sw.BASA_OK
        assert torch.equal(out, ref), (grid, win)


@pytest.mark.gpu
def test_noalloc_routes_equal_workspace_routes_at_full_size():
    # the routing configuration the benchmark times (Wan-like 720p, 40 heads,
    # 45 windows, d = 128: 1.8 MB of descriptors), called twice in a row with
    # the two shifts of the alternating pair
    wl = BY_NAME["wan-720p-21x45x80-w7x15x16"]
    q, k, _ = make_qkv(wl, device="cuda")
    for shift in wl.shifts:
        out = torch.empty((wl.B, wl.heads, sw.n_windows(wl.grid, wl.win)), dtype=torch.int32, device=q.device)
        assert _noalloc(q, k, wl.grid, wl.win, shift, 1, out) == sw.BASA_OK
        ref = sw.route(q, k, wl.grid, wl.win, shift, 1)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), shift


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4,097 window-heads of d = 128 need 4,097 * 128 * 8 bytes > 4 MiB; refused
    # on the host, before any device work (the pointers are never dereferenced)
    lib = sw._load()
    vp = ctypes.c_void_p
    a, r = vp(1 << 20), vp(1 << 34)
    rc = lib.basa_route_noalloc(a, a, 1, 4097, 1, 8, 8, 128, I3(1, 8, 8), I3(0, 0, 0), 1, r, None)
    assert rc == sw.BASA_ERR_SCRATCH_LIMIT
    assert "scratch" in sw.strerror(rc)
    # exactly at the limit the size check passes (the call then stops at the
    # misaligned q, the next check)
    assert 4096 * 128 * 2 * 4 == sw.ROUTE_NOALLOC_SCRATCH_BYTES
    m = vp((1 << 20) + 8)
    assert lib.basa_route_noalloc(m, a, 1, 4096, 1, 8, 8, 128, I3(1, 8, 8), I3(0, 0, 0), 1, r,
                                  None) == sw.BASA_ERR_ALIGNMENT
    assert lib.basa_route_noalloc(m, a, 1, 4097, 1, 8, 8, 128, I3(1, 8, 8), I3(0, 0, 0), 1, r,
                                  None) == sw.BASA_ERR_SCRATCH_LIMIT
