"""B200 (sm_100a) shifted local-window self-attention.

A thin ctypes binding over ``libbasa_swattn.so`` (C ABI in ``include/basa_swattn.h``).
Python only checks and marshals arguments; the roll, window gather, attention
and inverse roll all run in the CUDA kernel.  PyTorch supplies device memory
and streams.  There is no CPU fallback: if the library is missing or fails to
load, every call raises.

Method: "Backend-Agnostic Sparse Attention for Fast High-Resolution Visual
Generation" (BASA), §3.1 "Shifted Window Sparse Attention".
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "swattn_fwd", "swattn_fwd_from_host", "swattn_fwd_mem", "kv_pool", "kv_pool_tokens",
    "index_map", "index_map_host", "flops", "shift_schedule", "route", "route_workspace_bytes",
    "swattn_fwd_route", "route_noalloc", "n_windows",
    "last_device_error", "set_wait_timeout_ns", "strerror", "library_path", "SwattnError",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libbasa_swattn.so"
_lib = None
_lock = threading.Lock()
_I3 = ctypes.c_int * 3

BASA_OK = 0
BASA_ERR_INVALID_ARG = -1
BASA_ERR_UNSUPPORTED = -2
BASA_ERR_ALIGNMENT = -3
BASA_ERR_CUDA = -4
BASA_ERR_DEVICE = -5
BASA_ERR_ALIAS = -6
BASA_ERR_SCRATCH_LIMIT = -7
ROUTE_NOALLOC_SCRATCH_BYTES = 4 << 20


class SwattnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{_LIB_NAME} is not built ({path}); run "
                "`python -m shifted_window_attention_swattn_b200.build`")
        lib = ctypes.CDLL(path)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        lib.basa_swattn_fwd.argtypes = [vp, vp, vp, vp] + [ci] * 6 + [_I3, _I3, ctypes.c_float, vp]
        lib.basa_swattn_fwd.restype = ci
        lib.basa_swattn_index_map.argtypes = [ci, ci, ci, _I3, _I3, vp, vp]
        lib.basa_swattn_index_map.restype = ci
        lib.basa_swattn_index_map_host.argtypes = [ci, ci, ci, _I3, _I3, vp]
        lib.basa_swattn_index_map_host.restype = ci
        lib.basa_swattn_flops.argtypes = [ci] * 6 + [_I3, ctypes.POINTER(ctypes.c_double)]
        lib.basa_swattn_flops.restype = ci
        lib.basa_swattn_fwd_mem.argtypes = [vp] * 5 + [ci, vp] + [ci] * 6 + [_I3, _I3, ctypes.c_float, vp]
        lib.basa_swattn_fwd_mem.restype = ci
        lib.basa_kv_pool.argtypes = [vp] * 4 + [ci] * 6 + [_I3, vp]
        lib.basa_kv_pool.restype = ci
        lib.basa_kv_pool_tokens.argtypes = [ci, ci, ci, _I3, ctypes.POINTER(ctypes.c_int)]
        lib.basa_kv_pool_tokens.restype = ci
        lib.basa_shift_schedule.argtypes = [ci, _I3, _I3, vp]
        lib.basa_shift_schedule.restype = ci
        lib.basa_route_workspace_bytes.argtypes = [ci] * 6 + [_I3, ctypes.POINTER(ctypes.c_size_t)]
        lib.basa_route_workspace_bytes.restype = ci
        lib.basa_route.argtypes = [vp, vp] + [ci] * 6 + [_I3, _I3, ci, vp, ctypes.c_size_t, vp, vp]
        lib.basa_route.restype = ci
        lib.basa_route_noalloc.argtypes = [vp, vp] + [ci] * 6 + [_I3, _I3, ci, vp, vp]
        lib.basa_route_noalloc.restype = ci
        lib.basa_swattn_fwd_route.argtypes = [vp] * 6 + [ci, vp] + [ci] * 6 + [_I3, _I3, ctypes.c_float, vp]
        lib.basa_swattn_fwd_route.restype = ci
        lib.basa_swattn_last_device_error.argtypes = [vp]
        lib.basa_swattn_last_device_error.restype = ci
        lib.basa_swattn_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
        lib.basa_swattn_set_wait_timeout_ns.restype = ci
        lib.basa_swattn_set_test_stall.argtypes = [ci]
        lib.basa_swattn_set_test_stall.restype = ci
        lib.basa_strerror.argtypes = [ci]
        lib.basa_strerror.restype = ctypes.c_char_p
        _lib = lib
        return lib


def strerror(code: int) -> str:
    return _load().basa_strerror(int(code)).decode()


def _triple(x, what):
    t = tuple(int(a) for a in x)
    if len(t) != 3:
        raise ValueError(f"{what} must be a (t, h, w) triple")
    return t


def n_windows(grid, win) -> int:
    """Windows in the partition of ``grid`` by ``win``: the product of ceil(n_a / w_a)."""
    n = 1
    for extent, w in zip(_triple(grid, "grid"), _triple(win, "win")):
        if w < 1:
            raise ValueError("window extents must be >= 1")
        n *= -(-extent // w)
    return n


def _stream_handle(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _require_on(device, named):
    """Every (name, tensor) pair holds a CUDA tensor on ``device``: the kernels
    address all operands of a call on the GPU of its first input."""
    import torch
    for name, t in named:
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != device:
            where = t.device if isinstance(t, torch.Tensor) else type(t).__name__
            raise ValueError(f"{name} must be a CUDA tensor on {device} (got {where})")


def _call_on(device, fn, *args):
    """Calls the C entry point with ``device`` current (the library launches on
    the current device)."""
    import torch
    with torch.cuda.device(device):
        return fn(*args)


def swattn_fwd(q, k, v, grid, win, shift, scale=None, out=None, stream=None):
    """Shifted-window attention forward on device tensors.

    q, k, v: bf16 CUDA tensors [B, T*H*W, heads, d] (contiguous), grid = (T, H, W),
    win and shift (t, h, w) triples.  Returns ``out`` (allocated if not given).
    Asynchronous on ``stream`` (default: the current stream of q's device).
    """
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be contiguous [B, T*H*W, heads, d]")
    if q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must have the same shape")
    B, N, heads, d = q.shape
    if N != T * H * W:
        raise ValueError(f"token count {N} != T*H*W = {T * H * W}")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    _require_on(q.device, (("k", k), ("v", v), ("out", out)))
    if scale is None:
        scale = d ** -0.5
    rc = _call_on(q.device, lib.basa_swattn_fwd, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                  B, heads, T, H, W, d, _I3(*w3), _I3(*s3), float(scale), _stream_handle(stream, q.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_fwd")
    return out


def swattn_fwd_mem(q, k, v, kx, vx, grid, win, shift, scale=None, out=None, stream=None):
    """Shifted-window attention whose every window also attends to an extra K/V
    segment (§3.2): kx, vx are bf16 CUDA tensors [B, E, heads, d] (pooled memory
    from ``kv_pool``, other shared tokens, or both concatenated along dim 1)."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    for name, t in (("q", q), ("k", k), ("v", v), ("kx", kx), ("vx", vx)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be contiguous and 4-D")
    if q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must have the same shape")
    B, N, heads, d = q.shape
    if kx.shape != vx.shape or kx.shape[0] != B or kx.shape[2:] != q.shape[2:]:
        raise ValueError("kx, vx must be [B, E, heads, d] like q")
    if N != T * H * W:
        raise ValueError(f"token count {N} != T*H*W = {T * H * W}")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    _require_on(q.device, (("k", k), ("v", v), ("kx", kx), ("vx", vx), ("out", out)))
    if scale is None:
        scale = d ** -0.5
    E = kx.shape[1]
    rc = _call_on(q.device, lib.basa_swattn_fwd_mem, q.data_ptr(), k.data_ptr(), v.data_ptr(), kx.data_ptr(),
                  vx.data_ptr(), E, out.data_ptr(), B, heads, T, H, W, d, _I3(*w3), _I3(*s3), float(scale),
                  _stream_handle(stream, q.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_fwd_mem")
    return out


def _check_qkv(named, grid):
    import torch
    for name, t in named:
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be contiguous and 4-D")
    q = named[0][1]
    for name, t in named[1:]:
        if t.shape != q.shape:
            raise ValueError(f"{name} must have the shape of q")
    T, H, W = grid
    if q.shape[1] != T * H * W:
        raise ValueError(f"token count {q.shape[1]} != T*H*W = {T * H * W}")


def route_workspace_bytes(B, heads, grid, d, win) -> int:
    """Device bytes ``route`` needs for the fp32 window descriptors."""
    lib = _load()
    T, H, W = _triple(grid, "grid")
    n = ctypes.c_size_t(0)
    rc = lib.basa_route_workspace_bytes(int(B), int(heads), T, H, W, int(d), _I3(*_triple(win, "win")),
                                        ctypes.byref(n))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_route_workspace_bytes")
    return int(n.value)


def route(q, k, grid, win, shift, radius=1, out=None, workspace=None, stream=None):
    """Top-1 true-window routing (§3.3): int32 CUDA tensor [B, heads, n_windows],
    the routed window of every window of the shifted partition (-1: none).
    q, k: bf16 CUDA tensors [B, T*H*W, heads, d].  ``workspace`` (a CUDA tensor of
    at least ``route_workspace_bytes`` bytes) is allocated when not given."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    _check_qkv((("q", q), ("k", k)), (T, H, W))
    B, _, heads, d = q.shape
    nw = n_windows(grid, win)
    need = route_workspace_bytes(B, heads, grid, d, win)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    elif not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if out is None:
        out = torch.empty((B, heads, nw), dtype=torch.int32, device=q.device)
    elif out.shape != (B, heads, nw) or out.dtype != torch.int32 or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous int32 tensor of shape {(B, heads, nw)}")
    _require_on(q.device, (("k", k), ("workspace", workspace), ("out", out)))
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = _call_on(q.device, lib.basa_route, q.data_ptr(), k.data_ptr(), B, heads, T, H, W, d, _I3(*w3),
                  _I3(*s3), int(radius), workspace.data_ptr(), ws_bytes, out.data_ptr(),
                  _stream_handle(stream, q.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_route")
    return out


def route_noalloc(q, k, grid, win, shift, radius=1, out=None, stream=None):
    """``route`` through basa_route_noalloc: the library keeps the window
    descriptors in its own fixed device array, so the C call allocates nothing
    (for callers that cannot allocate at routing time).  Problems whose
    descriptors exceed ROUTE_NOALLOC_SCRATCH_BYTES raise SwattnError
    (BASA_ERR_SCRATCH_LIMIT).  Calls that can overlap on the GPU race on the
    shared array.  ``out`` (int32 [B, heads, n_windows]) is allocated here when
    not given."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    _check_qkv((("q", q), ("k", k)), (T, H, W))
    B, _, heads, d = q.shape
    nw = n_windows(grid, win)
    if out is None:
        out = torch.empty((B, heads, nw), dtype=torch.int32, device=q.device)
    elif out.shape != (B, heads, nw) or out.dtype != torch.int32 or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous int32 tensor of shape {(B, heads, nw)}")
    _require_on(q.device, (("k", k), ("out", out)))
    rc = _call_on(q.device, lib.basa_route_noalloc, q.data_ptr(), k.data_ptr(), B, heads, T, H, W, d, _I3(*w3),
                  _I3(*s3), int(radius), out.data_ptr(), _stream_handle(stream, q.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_route_noalloc")
    return out


def swattn_fwd_route(q, k, v, routed, grid, win, shift, kx=None, vx=None, scale=None, out=None, stream=None):
    """Shifted-window attention over S_i = W_i u R_i u G (§3.3): every window
    attends to its own tokens, to those of its routed window (``routed``: int32
    CUDA tensor [B, heads, n_windows] from ``route``; -1 = none) and, when given,
    to the extra K/V segment kx, vx (bf16 [B, E, heads, d], e.g. the pooled memory)."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    _check_qkv((("q", q), ("k", k), ("v", v)), (T, H, W))
    B, N, heads, d = q.shape
    nw = n_windows(grid, win)
    if (not isinstance(routed, torch.Tensor) or not routed.is_cuda or routed.dtype != torch.int32 or
            not routed.is_contiguous() or routed.numel() != B * heads * nw):
        raise ValueError(f"routed must be a contiguous int32 CUDA tensor of {B * heads * nw} entries")
    if (kx is None) != (vx is None):
        raise ValueError("give both kx and vx, or neither")
    E = 0
    if kx is not None:
        for name, t in (("kx", kx), ("vx", vx)):
            if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
                raise TypeError(f"{name} must be a bf16 CUDA tensor")
            if not t.is_contiguous() or t.dim() != 4:
                raise ValueError(f"{name} must be contiguous and 4-D")
        if kx.shape != vx.shape or kx.shape[0] != B or kx.shape[2:] != q.shape[2:]:
            raise ValueError("kx, vx must be [B, E, heads, d] like q")
        E = kx.shape[1]
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    named = [("k", k), ("v", v), ("routed", routed), ("out", out)]
    if E:
        named += [("kx", kx), ("vx", vx)]
    _require_on(q.device, named)
    if scale is None:
        scale = d ** -0.5
    rc = _call_on(q.device, lib.basa_swattn_fwd_route, q.data_ptr(), k.data_ptr(), v.data_ptr(), routed.data_ptr(),
                  kx.data_ptr() if E else None, vx.data_ptr() if E else None, E, out.data_ptr(), B, heads,
                  T, H, W, d, _I3(*w3), _I3(*s3), float(scale), _stream_handle(stream, q.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_fwd_route")
    return out


def kv_pool_tokens(grid, pool) -> int:
    """Pooled tokens G = prod ceil(n_a / pool_a) (§3.2)."""
    lib = _load()
    T, H, W = _triple(grid, "grid")
    G = ctypes.c_int(0)
    rc = lib.basa_kv_pool_tokens(T, H, W, _I3(*_triple(pool, "pool")), ctypes.byref(G))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_kv_pool_tokens")
    return G.value


def kv_pool(k, v, grid, pool, stream=None):
    """Pooled global memory (§3.2): (kbar, vbar), bf16 [B, G, heads, d] patch means of
    k and v over the unshifted grid, patches of pool = (p_t, p_h, p_w) in raster order."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    p3 = _triple(pool, "pool")
    for name, t in (("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be contiguous [B, T*H*W, heads, d]")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    B, N, heads, d = k.shape
    if N != T * H * W:
        raise ValueError(f"token count {N} != T*H*W = {T * H * W}")
    _require_on(k.device, (("v", v),))
    G = kv_pool_tokens(grid, p3)
    kbar = torch.empty((B, G, heads, d), dtype=torch.bfloat16, device=k.device)
    vbar = torch.empty_like(kbar)
    rc = _call_on(k.device, lib.basa_kv_pool, k.data_ptr(), v.data_ptr(), kbar.data_ptr(), vbar.data_ptr(), B,
                  heads, T, H, W, d, _I3(*p3), _stream_handle(stream, k.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_kv_pool")
    return kbar, vbar


def swattn_fwd_from_host(q_host, k_host, v_host, grid, win, shift, scale=None, out_host=None,
                         device="cuda", stream=None, dev_bufs=None):
    """The same forward for inputs in host memory: H2D copy, kernel, D2H copy.

    q_host, k_host, v_host: bf16 CPU tensors (pinned for asynchronous copies).
    ``dev_bufs`` = (q, k, v, out) device tensors may be passed to reuse memory.
    Returns the host output tensor; the call synchronises the stream.
    """
    import torch
    if dev_bufs is None:
        dev_bufs = tuple(torch.empty(q_host.shape, dtype=torch.bfloat16, device=device)
                         for _ in range(4))
    qd, kd, vd, od = dev_bufs
    if stream is None:
        stream = torch.cuda.current_stream(qd.device)
    with torch.cuda.stream(stream):
        qd.copy_(q_host, non_blocking=True)
        kd.copy_(k_host, non_blocking=True)
        vd.copy_(v_host, non_blocking=True)
        swattn_fwd(qd, kd, vd, grid, win, shift, scale, out=od, stream=stream)
        if out_host is None:
            out_host = torch.empty(q_host.shape, dtype=torch.bfloat16, pin_memory=True)
        out_host.copy_(od, non_blocking=True)
    stream.synchronize()
    return out_host


def index_map(grid, win, shift, device="cuda", stream=None):
    """Device-computed token_of_slot [n_windows, w_t*w_h*w_w] int32 (-1 padded)."""
    import torch
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    if min(w3) < 1 or min(T, H, W) < 1:
        raise ValueError("extents must be >= 1")
    nwin = 1
    for n, w in zip((T, H, W), w3):
        nwin *= -(-n // w)
    out = torch.empty((nwin, w3[0] * w3[1] * w3[2]), dtype=torch.int32, device=device)
    rc = _call_on(out.device, lib.basa_swattn_index_map, T, H, W, _I3(*w3), _I3(*s3), out.data_ptr(),
                  _stream_handle(stream, out.device))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_index_map")
    return out


def index_map_host(grid, win, shift):
    """Host-computed token_of_slot (same source function as the kernel's)."""
    import numpy as np
    lib = _load()
    T, H, W = _triple(grid, "grid")
    w3, s3 = _triple(win, "win"), _triple(shift, "shift")
    if min(w3) < 1 or min(T, H, W) < 1:
        raise SwattnError(BASA_ERR_INVALID_ARG, "basa_swattn_index_map_host")
    nwin = 1
    for n, w in zip((T, H, W), w3):
        nwin *= -(-n // w)
    out = np.empty((nwin, w3[0] * w3[1] * w3[2]), dtype=np.int32)
    rc = lib.basa_swattn_index_map_host(T, H, W, _I3(*w3), _I3(*s3), out.ctypes.data)
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_index_map_host")
    return out


def flops(B, heads, grid, d, win) -> float:
    """Algorithmic FLOPs of one forward: sum over windows of 4 n_m^2 d, times B*heads."""
    lib = _load()
    T, H, W = _triple(grid, "grid")
    res = ctypes.c_double(0.0)
    rc = lib.basa_swattn_flops(int(B), int(heads), T, H, W, int(d), _I3(*_triple(win, "win")),
                               ctypes.byref(res))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_swattn_flops")
    return res.value


def shift_schedule(L, win, step_offset=(0, 0, 0)):
    """Per-layer shifts of the interleaved shift schedule (§3.1): a list of L
    (t, h, w) triples for layers 0..L-1, each usable as ``swattn_fwd``'s ``shift``.
    ``step_offset`` is the schedule's denoising-step term c_s."""
    lib = _load()
    w3, c3 = _triple(win, "win"), _triple(step_offset, "step_offset")
    L = int(L)
    if L < 1:
        raise SwattnError(BASA_ERR_INVALID_ARG, "basa_shift_schedule")
    out = (ctypes.c_int * (3 * L))()
    rc = lib.basa_shift_schedule(L, _I3(*w3), _I3(*c3), ctypes.cast(out, ctypes.c_void_p))
    if rc != BASA_OK:
        raise SwattnError(rc, "basa_shift_schedule")
    return [tuple(out[3 * l:3 * l + 3]) for l in range(L)]


def last_device_error(stream=None) -> int:
    """Synchronise and return (and clear) the device-side wait-timeout record."""
    import torch
    return _load().basa_swattn_last_device_error(
        _stream_handle(stream, torch.device("cuda", torch.cuda.current_device())))


def set_wait_timeout_ns(ns: int) -> None:
    _load().basa_swattn_set_wait_timeout_ns(int(ns))


def set_test_stall(on: bool) -> None:
    """Test hook: make every launch's MMA issuer wait on a barrier nothing arrives on."""
    _load().basa_swattn_set_test_stall(1 if on else 0)
