"""fp64 CPU oracle for shifted local-window self-attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``shifted_window_attention_swattn_b200``) never imports it and shares no
code with it.

The arithmetic lives in ``ref_swattn.c`` (plain C, fp64, one materialised array
per stage), including the pooled global memory of §3.2 ("K/V-Pooled Global
Memory") and the true-window routing of §3.3 ("Content-Adaptive True-Window
Routing").  This module only builds that file with gcc and marshals arguments
through ctypes.  Method: "Backend-Agnostic Sparse Attention for Fast
High-Resolution Visual Generation" (BASA), §3.1 "Shifted Window Sparse
Attention" and Appendix A.1 "Regular execution with standard attention
backends".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ref_swattn.c")
_LIB_PATH = os.path.join(_HERE, "libref_swattn.so")
_lib = None
_lock = threading.Lock()

_I3 = ctypes.c_int * 3


def build(force: bool = False) -> str:
    """Compile ref_swattn.c into libref_swattn.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-Wall", "-fPIC", "-shared",
             "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oref_index_map.argtypes = [ctypes.c_int] * 3 + [_I3, _I3, ctypes.c_void_p, ctypes.c_void_p]
            lib.oref_index_map.restype = ctypes.c_int
            lib.oref_swattn_fwd.argtypes = (
                [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [_I3, _I3, ctypes.c_double]
                + [ctypes.c_int] * 3)
            lib.oref_swattn_fwd.restype = ctypes.c_int
            lib.oref_swattn_rows.argtypes = (
                [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [_I3, _I3, ctypes.c_double]
                + [ctypes.c_void_p, ctypes.c_long, ctypes.c_void_p])
            lib.oref_swattn_rows.restype = ctypes.c_int
            lib.oref_flops.argtypes = [ctypes.c_int] * 6 + [_I3]
            lib.oref_flops.restype = ctypes.c_double
            lib.oref_swattn_fwd_mem.argtypes = (
                [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 6
                + [_I3, _I3, ctypes.c_double] + [ctypes.c_int] * 3)
            lib.oref_swattn_fwd_mem.restype = ctypes.c_int
            lib.oref_kv_pool.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 6 + [_I3]
            lib.oref_kv_pool.restype = ctypes.c_int
            lib.oref_route.argtypes = ([ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 6 +
                                       [_I3, _I3, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p])
            lib.oref_route.restype = ctypes.c_int
            lib.oref_swattn_fwd_route.argtypes = (
                [ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 6 +
                [_I3, _I3, ctypes.c_double])
            lib.oref_swattn_fwd_route.restype = ctypes.c_int
            lib.oref_swattn_rows_route.argtypes = (
                [ctypes.c_void_p] * 6 + [ctypes.c_int] + [ctypes.c_int] * 6 +
                [_I3, _I3, ctypes.c_double, ctypes.c_void_p, ctypes.c_long, ctypes.c_void_p])
            lib.oref_swattn_rows_route.restype = ctypes.c_int
            _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 data as a contiguous uint16 numpy array of bit patterns.

    Accepts a torch bf16 tensor (any device) or a uint16 numpy array.
    """
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy input must hold bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch  # local: the oracle itself needs only numpy
    if x.dtype != torch.bfloat16:
        raise TypeError("torch input must be bfloat16")
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _geom_args(win, shift):
    if len(win) != 3 or len(shift) != 3:
        raise ValueError("win and shift are (t, h, w) triples")
    return _I3(*[int(a) for a in win]), _I3(*[int(a) for a in shift])


def n_windows(T, H, W, win) -> int:
    """Windows in the grid: ceil(n_a / w_a) per axis (truncated last windows)."""
    n = 1
    for ext, w in zip((T, H, W), win):
        if int(w) < 1 or int(ext) < 1:
            raise ValueError("grid and window extents must be >= 1")
        n *= -(-int(ext) // int(w))
    return n


def index_map(T, H, W, win, shift):
    """(token_of_slot [n_windows, w_t*w_h*w_w] int32 with -1 padding, count [n_windows])."""
    lib = _load()
    nw = n_windows(T, H, W, win)
    nmax = int(win[0]) * int(win[1]) * int(win[2])
    tos = np.empty((nw, nmax), dtype=np.int32)
    cnt = np.empty((nw,), dtype=np.int32)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_index_map(int(T), int(H), int(W), w3, s3, tos.ctypes.data, cnt.ctypes.data)
    if rc != 0:
        raise ValueError(f"oref_index_map failed ({rc})")
    return tos, cnt


def swattn_fwd(q, k, v, B, heads, T, H, W, d, win, shift, scale, head_range=None, nthreads=None):
    """fp64 output [B, T*H*W, heads, d] of the shifted-window forward.

    Heads outside ``head_range`` (default: all) are left as NaN.
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N = int(T) * int(H) * int(W)
    expect = int(B) * N * int(heads) * int(d)
    for a in (qb, kb, vb):
        if a.size != expect:
            raise ValueError("q/k/v must hold B*T*H*W*heads*d elements")
    h0, h1 = (0, int(heads)) if head_range is None else (int(head_range[0]), int(head_range[1]))
    if nthreads is None:
        nthreads = max(1, len(os.sched_getaffinity(0)))
    out = np.full((int(B), N, int(heads), int(d)), np.nan, dtype=np.float64)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_swattn_fwd(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, out.ctypes.data,
                             int(B), int(heads), int(T), int(H), int(W), int(d), w3, s3,
                             float(scale), h0, h1, int(nthreads))
    if rc != 0:
        raise ValueError(f"oref_swattn_fwd failed ({rc})")
    return out


def swattn_rows(q, k, v, B, heads, T, H, W, d, win, shift, scale, triples):
    """fp64 output rows [len(triples), d] for (b, token, head) triples."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    tr = np.ascontiguousarray(np.asarray(triples, dtype=np.int64).reshape(-1, 3))
    out = np.empty((tr.shape[0], int(d)), dtype=np.float64)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_swattn_rows(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                              int(B), int(heads), int(T), int(H), int(W), int(d), w3, s3,
                              float(scale), tr.ctypes.data, tr.shape[0], out.ctypes.data)
    if rc != 0:
        raise ValueError(f"oref_swattn_rows failed ({rc})")
    return out


def flops(B, heads, T, H, W, d, win) -> float:
    """Algorithmic FLOPs: sum over windows of 4 * n_m^2 * d, times B * heads."""
    lib = _load()
    w3 = _I3(*[int(a) for a in win])
    return float(lib.oref_flops(int(B), int(heads), int(T), int(H), int(W), int(d), w3))


def n_pooled(T, H, W, pool) -> int:
    """Pooled memory tokens G = prod ceil(n_a / p_a) (§3.2; truncated last patches)."""
    n = 1
    for ext, p in zip((T, H, W), pool):
        if int(p) < 1 or int(ext) < 1:
            raise ValueError("grid and pooling extents must be >= 1")
        n *= -(-int(ext) // int(p))
    return n


def kv_pool(x, B, heads, T, H, W, d, pool):
    """fp64 [B, G, heads, d]: means of x (bf16 [B, T*H*W, heads, d]) over the
    p_t x p_h x p_w patches of the unshifted grid, patches in raster order (§3.2)."""
    lib = _load()
    xb = _bits(x)
    G = n_pooled(T, H, W, pool)
    out = np.empty((int(B), G, int(heads), int(d)), dtype=np.float64)
    rc = lib.oref_kv_pool(xb.ctypes.data, out.ctypes.data, int(B), int(heads), int(T), int(H),
                          int(W), int(d), _I3(*[int(a) for a in pool]))
    if rc != 0:
        raise ValueError(f"oref_kv_pool failed ({rc})")
    return out


def round_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values to bf16 (round to nearest, ties to even) as uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def swattn_fwd_mem(q, k, v, kx, vx, E, B, heads, T, H, W, d, win, shift, scale, nthreads=None):
    """fp64 [B, T*H*W, heads, d]: the shifted-window forward where every window's
    keys and values are extended by the E extra tokens kx, vx (bf16 [B, E, heads, d])
    of its (b, head): K^mem = [K_W; K_x], V^mem = [V_W; V_x] (§3.2)."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    kxb, vxb = _bits(kx), _bits(vx)
    N = int(T) * int(H) * int(W)
    if kxb.size != int(B) * int(E) * int(heads) * int(d) or vxb.size != kxb.size:
        raise ValueError("kx/vx must hold B*E*heads*d elements")
    if nthreads is None:
        nthreads = max(1, len(os.sched_getaffinity(0)))
    out = np.full((int(B), N, int(heads), int(d)), np.nan, dtype=np.float64)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_swattn_fwd_mem(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, kxb.ctypes.data,
                                 vxb.ctypes.data, int(E), out.ctypes.data, int(B), int(heads),
                                 int(T), int(H), int(W), int(d), w3, s3, float(scale), 0,
                                 int(heads), int(nthreads))
    if rc != 0:
        raise ValueError(f"oref_swattn_fwd_mem failed ({rc})")
    return out


def route(q, k, B, heads, T, H, W, d, win, shift, radius=1, with_scores=False):
    """int32 [B, heads, n_windows]: the routed window of every window of the
    (shifted) partition, -1 where a window has no candidate (§3.3: top-1 of
    s_ij = q_i k_j^T / sqrt(d) over the other windows of the same temporal
    index within spatial window distance `radius`).  With with_scores, also
    the fp64 scores [B, heads, n_windows, n_windows] (-inf off the candidates)."""
    lib = _load()
    qb, kb = _bits(q), _bits(k)
    nw = n_windows(T, H, W, win)
    routed = np.full((int(B), int(heads), nw), -2, dtype=np.int32)
    scores = np.full((int(B), int(heads), nw, nw), np.nan) if with_scores else None
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_route(qb.ctypes.data, kb.ctypes.data, int(B), int(heads), int(T), int(H), int(W),
                        int(d), w3, s3, int(radius), routed.ctypes.data,
                        scores.ctypes.data if with_scores else None)
    if rc != 0:
        raise ValueError(f"oref_route failed ({rc})")
    return (routed, scores) if with_scores else routed


def swattn_fwd_route(q, k, v, routed, kx, vx, E, B, heads, T, H, W, d, win, shift, scale):
    """fp64 [B, T*H*W, heads, d]: every window attends to its own tokens, the
    tokens of its routed window (routed int32 [B, heads, n_windows], -1 = none)
    and the E extra tokens kx, vx (bf16 [B, E, heads, d]; E may be 0):
    the key/value source S_i = W_i u R_i u G of §3.3."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    nw = n_windows(T, H, W, win)
    rt = np.ascontiguousarray(np.asarray(routed, dtype=np.int32))
    if rt.size != int(B) * int(heads) * nw:
        raise ValueError("routed must hold B*heads*n_windows entries")
    if int(E) > 0:
        kxb, vxb = _bits(kx), _bits(vx)
        if kxb.size != int(B) * int(E) * int(heads) * int(d) or vxb.size != kxb.size:
            raise ValueError("kx/vx must hold B*E*heads*d elements")
        kxp, vxp = kxb.ctypes.data, vxb.ctypes.data
    else:
        kxp = vxp = None
    N = int(T) * int(H) * int(W)
    out = np.full((int(B), N, int(heads), int(d)), np.nan, dtype=np.float64)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_swattn_fwd_route(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, rt.ctypes.data,
                                   kxp, vxp, int(E), out.ctypes.data, int(B), int(heads), int(T),
                                   int(H), int(W), int(d), w3, s3, float(scale))
    if rc != 0:
        raise ValueError(f"oref_swattn_fwd_route failed ({rc})")
    return out


def swattn_rows_route(q, k, v, routed, kx, vx, E, B, heads, T, H, W, d, win, shift, scale, triples):
    """fp64 rows [len(triples), d] of ``swattn_fwd_route`` for (b, token, head) triples."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    rt = np.ascontiguousarray(np.asarray(routed, dtype=np.int32))
    if rt.size != int(B) * int(heads) * n_windows(T, H, W, win):
        raise ValueError("routed must hold B*heads*n_windows entries")
    if int(E) > 0:
        kxb, vxb = _bits(kx), _bits(vx)
        if kxb.size != int(B) * int(E) * int(heads) * int(d) or vxb.size != kxb.size:
            raise ValueError("kx/vx must hold B*E*heads*d elements")
        kxp, vxp = kxb.ctypes.data, vxb.ctypes.data
    else:
        kxp = vxp = None
    tr = np.ascontiguousarray(np.asarray(triples, dtype=np.int64).reshape(-1, 3))
    out = np.empty((tr.shape[0], int(d)), dtype=np.float64)
    w3, s3 = _geom_args(win, shift)
    rc = lib.oref_swattn_rows_route(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, rt.ctypes.data, kxp, vxp,
                                    int(E), int(B), int(heads), int(T), int(H), int(W), int(d), w3, s3,
                                    float(scale), tr.ctypes.data, tr.shape[0], out.ctypes.data)
    if rc != 0:
        raise ValueError(f"oref_swattn_rows_route failed ({rc})")
    return out


def shift_schedule(L, win, step_offset=(0, 0, 0)):
    """Interleaved shift schedule, §3.1 "Interleaved shift schedule", taken step
    by step in the pages' order for each axis with window w:

      delta = max(1, floor(w / L));  a_i = (i * delta) mod w, i = 0..L-1;
      b = (a_0, a_K, a_1, a_{K+1}, ..., a_{K-1}, a_{L-1}): the halves
          a_0..a_{K-1} and a_K..a_{L-1} interleaved, first half first;
      Delta_l = (b_l + c_s) mod w.

    Readings: K = ceil(L / 2) (the pages do not define K; this is the value for
    which the printed sequence ends with a_{K-1}, a_{L-1} when L is even), and
    for odd L the first half's extra element a_{K-1} comes last.  c_s, the
    denoising-step offset, is an input (the pages leave its values open).
    Returns a list of L (t, h, w) triples.
    """
    L = int(L)
    if L < 1 or len(win) != 3 or min(win) < 1:
        raise ValueError("L and the window extents must be >= 1")
    K = -(-L // 2)
    per_axis = []
    for w, c in zip(win, step_offset):
        delta = max(1, w // L)
        a = [(i * delta) % w for i in range(L)]
        first, second = a[:K], a[K:]
        b = []
        for i in range(K):
            b.append(first[i])
            if i < len(second):
                b.append(second[i])
        per_axis.append([(x + c) % w for x in b])
    return [tuple(per_axis[ax][l] for ax in range(3)) for l in range(L)]
