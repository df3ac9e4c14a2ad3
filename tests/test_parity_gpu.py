"""GPU parity: the sm_100a kernel against the fp64 oracle, through the C ABI.

Tolerances (bf16 inputs, fp32 accumulation, P and the output rounded to bf16):
max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the oracle, over
every compared element.  Index maps must match exactly.

Small cases compare every output element; the full-size workloads compare
sampled rows that the oracle computes one by one, in the same launch
configuration the benchmark times.
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import shifted_window_attention_swattn_b200 as sw
from shifted_window_attention_swattn_b200.inputs import BY_NAME, WORKLOADS, make_custom, make_qkv

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def _check(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert err.max() <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={err.max():.3e} rel_l2={rel:.3e}"
    return err.max(), rel


def _run_gpu(q, k, v, grid, win, shift, scale):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = sw.swattn_fwd(qd, kd, vd, grid, win, shift, scale)
    assert sw.last_device_error() == sw.BASA_OK
    return out


def _full_compare_inputs(q, k, v, B, heads, d, grid, win, shift, scale):
    T, H, W = grid
    out = _run_gpu(q, k, v, grid, win, shift, scale).float().cpu().numpy()
    ref = oracle.swattn_fwd(q, k, v, B, heads, T, H, W, d, win, shift, scale)
    return _check(out, ref, f"grid={grid} win={win} shift={shift} d={d}")


def _full_compare(B, heads, d, grid, win, shift, scale=None, seed=0, dist="normal"):
    T, H, W = grid
    q, k, v = make_custom(B, heads, d, T, H, W, seed, dist=dist)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = _run_gpu(q, k, v, grid, win, shift, scale).float().cpu().numpy()
    ref = oracle.swattn_fwd(q, k, v, B, heads, T, H, W, d, win, shift, scale)
    return _check(out, ref, f"grid={grid} win={win} shift={shift} d={d}")


# ---------------------------------------------------------------- index maps

@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_device_index_map_exact_on_workloads(wl):
    for shift in wl.shifts:
        got = sw.index_map(wl.grid, wl.win, shift).cpu().numpy()
        ref, _ = oracle.index_map(*wl.grid, wl.win, shift)
        assert np.array_equal(got, ref), shift


@pytest.mark.parametrize("grid,win,shift", [
    ((3, 1, 5), (2, 1, 2), (1, 0, 2)),
    ((5, 9, 11), (2, 4, 5), (1, 7, -3)),
    ((1, 20, 28), (1, 7, 9), (0, 3, 5)),
])
def test_device_index_map_exact_ragged(grid, win, shift):
    got = sw.index_map(grid, win, shift).cpu().numpy()
    ref, _ = oracle.index_map(*grid, win, shift)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- small, every element

@pytest.mark.parametrize("shift", [(0, 0, 0), (0, 4, 4)])
def test_tiny_2d_workload(shift):
    wl = WORKLOADS[0]
    q, k, v = make_qkv(wl)
    out = _run_gpu(q, k, v, wl.grid, wl.win, shift, wl.scale).float().cpu().numpy()
    ref = oracle.swattn_fwd(q, k, v, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, wl.scale)
    _check(out, ref, f"tiny shift={shift}")


@pytest.mark.parametrize("B,heads,d,grid,win,shift", [
    (2, 3, 128, (1, 20, 28), (1, 7, 9), (0, 3, 5)),      # n_w = 63, truncated windows
    (1, 2, 64, (5, 9, 11), (2, 4, 5), (1, 7, -3)),       # 3D, truncation on every axis
    (1, 2, 128, (1, 24, 24), (1, 12, 13), (0, 6, 11)),   # n_w = 156: two ragged tiles
    (1, 2, 128, (2, 16, 20), (2, 16, 10), (1, 8, 5)),    # n_w = 320: tiles 128+128+64
    (1, 1, 128, (1, 4, 300), (1, 1, 300), (0, 1, 77)),   # 300-token row windows
    (1, 2, 64, (1, 16, 16), (1, 8, 16), (0, 3, 9)),      # exactly 128 tokens
    (1, 2, 128, (1, 3, 43), (1, 3, 43), (0, 1, 20)),     # 129 tokens
    (3, 1, 64, (2, 6, 6), (1, 3, 3), (1, 1, 2)),         # B = 3
    (1, 4, 128, (3, 10, 13), (3, 5, 13), (2, 4, 6)),     # 195 tokens, 3D
])
def test_ragged_and_edge_shapes(B, heads, d, grid, win, shift):
    _full_compare(B, heads, d, grid, win, shift, seed=B * 100 + d)


def test_full_attention_mode_tiny():
    wl = WORKLOADS[0]
    _full_compare(1, 2, 64, wl.grid, wl.grid, (0, 0, 0), seed=3)


def test_sharp_softmax_exercises_rescaling():
    # scale 1 with d = 128 gives logits of std ~11: the running max moves a lot.
    _full_compare(1, 2, 128, (1, 24, 24), (1, 12, 12), (0, 6, 6), scale=1.0, seed=21)


@pytest.mark.parametrize("d", [128, 64])
def test_logits_jump_by_hundreds_between_key_tiles(d):
    # keys of the window's later key tiles are planted as large multiples of
    # their query, so the row maximum grows by far more than fp32 exponents
    # span (~2^130) from one key tile to the next: the running maximum must
    # move (O rescaled) without any intermediate overflow
    grid, win, shift = (1, 24, 24), (1, 24, 12), (0, 0, 5)     # 288-token windows: tiles 0-127, 128-255, 256-287
    q, k, v = make_custom(1, 2, d, *grid, seed=40 + d)
    tos, cnt = oracle.index_map(*grid, win, shift)
    rng = np.random.default_rng(d)
    for wid in range(tos.shape[0]):
        for slot in (150, 200, 270):
            tok = int(tos[wid, slot])
            src = int(tos[wid, int(rng.integers(0, 128))])     # a query of the first tile
            k[0, tok] = (q[0, src].float() * (4.0 if slot < 256 else 8.0)).to(torch.bfloat16)
    _full_compare_inputs(q, k, v, 1, 2, d, grid, win, shift, 1.0 / math.sqrt(d))


def test_uniform_inputs():
    _full_compare(1, 2, 128, (2, 12, 12), (2, 6, 12), (1, 3, 5), seed=22, dist="uniform")


def test_single_token_windows_return_v():
    T, H, W = 2, 3, 8
    q, k, v = make_custom(1, 2, 64, T, H, W, 5)
    out = _run_gpu(q, k, v, (T, H, W), (1, 1, 1), (1, 2, 3), 0.125)
    assert torch.equal(out.cpu(), v)


def test_scale_zero_gives_window_mean():
    _full_compare(1, 2, 128, (1, 12, 20), (1, 6, 10), (0, 2, 7), scale=0.0, seed=23)


def test_shift_by_grid_extent_matches_reduced_shift():
    T, H, W = 1, 16, 16
    q, k, v = make_custom(1, 2, 128, T, H, W, 7)
    a = _run_gpu(q, k, v, (T, H, W), (1, 8, 8), (0, 3, 5), 0.09)
    b = _run_gpu(q, k, v, (T, H, W), (1, 8, 8), (5, 3 - 2 * H, 5 + W), 0.09)
    assert torch.equal(a, b)


def test_repeated_calls_are_deterministic():
    T, H, W = 1, 32, 32
    q, k, v = make_custom(1, 4, 128, T, H, W, 8)
    a = _run_gpu(q, k, v, (T, H, W), (1, 16, 16), (0, 8, 8), 0.09)
    b = _run_gpu(q, k, v, (T, H, W), (1, 16, 16), (0, 8, 8), 0.09)
    assert torch.equal(a, b)


def test_host_buffer_entry_matches_device_entry():
    T, H, W = 1, 16, 32
    q, k, v = make_custom(1, 2, 128, T, H, W, 9)
    dev = _run_gpu(q, k, v, (T, H, W), (1, 8, 16), (0, 4, 8), 0.09).cpu()
    host = sw.swattn_fwd_from_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), (T, H, W),
                                   (1, 8, 16), (0, 4, 8), 0.09)
    assert torch.equal(dev, host)


def test_binding_rejects_operands_off_the_input_device():
    # a CPU output (or routes, workspace, extra segment) next to CUDA inputs is
    # refused before anything is launched
    grid, win, shift = (1, 16, 16), (1, 8, 8), (0, 4, 4)
    q, k, v = (t.cuda() for t in make_custom(1, 2, 128, *grid, seed=12))
    with pytest.raises(ValueError):
        sw.swattn_fwd(q, k, v, grid, win, shift, out=torch.empty(q.shape, dtype=torch.bfloat16))
    with pytest.raises((TypeError, ValueError)):
        sw.swattn_fwd_mem(q, k, v, k[:, :8].contiguous().cpu(), v[:, :8].contiguous(), grid, win, shift)
    with pytest.raises(ValueError):
        sw.route(q, k, grid, win, shift, out=torch.empty((1, 2, 4), dtype=torch.int32))
    with pytest.raises(ValueError):
        sw.route(q, k, grid, win, shift, workspace=torch.empty(1 << 16, dtype=torch.uint8))
    with pytest.raises(ValueError):
        sw.swattn_fwd_route(q, k, v, torch.full((1, 2, 4), -1, dtype=torch.int32), grid, win, shift)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- full-size workloads, sampled rows

def _sample_triples(wl, shift, n_random, rng):
    """Random (b, token, head) triples plus every query of one whole window."""
    tri = np.stack([rng.integers(0, wl.B, n_random), rng.integers(0, wl.N, n_random),
                    rng.integers(0, wl.heads, n_random)], axis=1)
    tos, cnt = oracle.index_map(*wl.grid, wl.win, shift)
    wid = int(rng.integers(0, tos.shape[0]))
    toks = tos[wid, :cnt[wid]]
    whole = np.stack([np.zeros_like(toks), toks, np.full_like(toks, wl.heads - 1)], axis=1)
    return np.concatenate([tri, whole]).astype(np.int64)


@pytest.mark.parametrize("wl", WORKLOADS[1:], ids=lambda w: w.name)
def test_full_size_workloads_sampled(wl):
    q, k, v = make_qkv(wl)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rng = np.random.default_rng(wl.seed)
    for shift in wl.shifts:
        out = sw.swattn_fwd(qd, kd, vd, wl.grid, wl.win, shift, wl.scale)
        assert sw.last_device_error() == sw.BASA_OK
        tri = _sample_triples(wl, shift, 1500, rng)
        ref = oracle.swattn_rows(q, k, v, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift,
                                 wl.scale, tri)
        got = out[tri[:, 0], tri[:, 1], tri[:, 2]].float().cpu().numpy()
        _check(got, ref, f"{wl.name} shift={shift}")
        assert torch.isfinite(out).all()
        del out


@pytest.mark.parametrize("wl", WORKLOADS[1:2], ids=lambda w: w.name)
def test_full_attention_mode_sampled(wl):
    q, k, v = make_qkv(wl)
    dev = torch.device("cuda:0")
    out = sw.swattn_fwd(q.to(dev), k.to(dev), v.to(dev), wl.grid, wl.grid, (0, 0, 0), wl.scale)
    assert sw.last_device_error() == sw.BASA_OK
    rng = np.random.default_rng(99)
    tri = np.stack([np.zeros(400, dtype=np.int64), rng.integers(0, wl.N, 400),
                    rng.integers(0, wl.heads, 400)], axis=1)
    ref = oracle.swattn_rows(q, k, v, wl.B, wl.heads, *wl.grid, wl.d, wl.grid, (0, 0, 0),
                             wl.scale, tri)
    got = out[tri[:, 0], tri[:, 1], tri[:, 2]].float().cpu().numpy()
    _check(got, ref, "full attention")


def _oracle_rows_threaded(fn, tri, *args):
    """fn(*args, triples) over chunks of `tri` on all host threads (the oracle's
    per-row C path releases the GIL); rows in the order of `tri`."""
    threads = max(1, len(os.sched_getaffinity(0)))
    chunks = [c for c in np.array_split(tri, threads * 2) if len(c)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(lambda c: fn(*args, c), chunks))
    return np.concatenate(parts)


# The full-attention mode at the sizes the benchmark times it (the denominator of
# the speedup over full attention): 65,536 to 131,040 keys per query, 512 to 1,024
# key steps per 512-query unit.  Random rows of every head, plus every query of
# the last 512-query unit of one head (ragged on two of the grids), so that whole
# long key loops, including the tail unit, are checked against fp64.
FULL_MODE_AT_BENCH_SIZE = [BY_NAME["flux-4096px-256x256-w32"], BY_NAME["wan-720p-21x45x80-w7x15x16"],
                           BY_NAME["wan-pages-21x60x104-w21x15x26"]]


@pytest.mark.parametrize("wl", FULL_MODE_AT_BENCH_SIZE, ids=lambda w: w.name)
def test_full_attention_mode_at_benchmark_size_sampled(wl):
    q, k, v = make_qkv(wl)
    dev = torch.device("cuda:0")
    out = sw.swattn_fwd(q.to(dev), k.to(dev), v.to(dev), wl.grid, wl.grid, (0, 0, 0), wl.scale)
    assert sw.last_device_error() == sw.BASA_OK
    rng = np.random.default_rng(wl.seed + 700)
    n_rand = 400
    tri = np.stack([rng.integers(0, wl.B, n_rand), rng.integers(0, wl.N, n_rand),
                    rng.integers(0, wl.heads, n_rand)], axis=1)
    q0 = ((wl.N - 1) // 512) * 512                      # first query of the last unit
    toks = np.arange(q0, wl.N)
    head = int(rng.integers(0, wl.heads))
    unit = np.stack([np.zeros_like(toks), toks, np.full_like(toks, head)], axis=1)
    tri = np.concatenate([tri, unit]).astype(np.int64)
    qb, kb, vb = oracle._bits(q), oracle._bits(k), oracle._bits(v)
    ref = _oracle_rows_threaded(oracle.swattn_rows, tri, qb, kb, vb, wl.B, wl.heads, *wl.grid, wl.d, wl.grid,
                                (0, 0, 0), wl.scale)
    got = out[tri[:, 0], tri[:, 1], tri[:, 2]].float().cpu().numpy()
    _check(got[:n_rand], ref[:n_rand], f"{wl.name} full attention, random rows")
    _check(got[n_rand:], ref[n_rand:], f"{wl.name} full attention, last unit of head {head}")
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("d,grid,win,L", [
    (128, (1, 24, 24), (1, 8, 8), 4),       # 2D, every layer of a 4-layer schedule
    (64, (3, 12, 10), (2, 6, 5), 3),        # 3D, truncated windows along t
    (128, (2, 9, 20), (2, 9, 7), 5),        # odd L, truncated along w
])
def test_shift_schedule_layers(d, grid, win, L):
    # every layer of the interleaved shift schedule, through the kernel, against the oracle
    T, H, W = grid
    q, k, v = make_custom(1, 2, d, T, H, W, seed=L)
    scale = 1.0 / math.sqrt(d)
    for shift in sw.shift_schedule(L, win, (0, 1, 2)):
        out = _run_gpu(q, k, v, grid, win, shift, scale).float().cpu().numpy()
        ref = oracle.swattn_fwd(q, k, v, 1, 2, T, H, W, d, win, shift, scale)
        _check(out, ref, f"schedule layer shift={shift}")


# ---------------------------------------------------------------- pooled global memory (§3.2)

@pytest.mark.parametrize("d,grid,pool", [
    (128, (1, 24, 24), (1, 4, 4)),
    (64, (3, 10, 13), (2, 4, 4)),       # temporal pooling, truncated patches along t, h, w
    (128, (2, 9, 20), (1, 3, 7)),
])
def test_kv_pool_matches_oracle(d, grid, pool):
    T, H, W = grid
    q, k, v = make_custom(2, 3, d, T, H, W, seed=sum(pool))
    kbar, vbar = sw.kv_pool(k.cuda(), v.cuda(), grid, pool)
    torch.cuda.synchronize()
    for got, x in ((kbar, k), (vbar, v)):
        ref = oracle.kv_pool(x, 2, 3, T, H, W, d, pool)
        g = got.float().cpu().numpy().astype(np.float64)
        # fp32 sums rounded to bf16 once: within half a bf16 ulp of the exact mean
        assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def _extra(B, E, heads, d, seed):
    kx, vx, _ = make_custom(B, heads, d, 1, 1, E, seed=seed)
    return kx, vx


@pytest.mark.parametrize("B,heads,d,grid,win,shift,E", [
    (1, 2, 128, (2, 9, 20), (2, 9, 7), (1, 4, 3), 37),       # pair kernel, one partial extra tile
    (1, 2, 128, (1, 24, 24), (1, 8, 8), (0, 4, 4), 300),     # three extra tiles, the last partial
    (2, 1, 128, (1, 16, 16), (1, 16, 16), (0, 0, 0), 128),   # full attention plus one exact extra tile
    (1, 2, 64, (3, 10, 13), (2, 4, 5), (1, 3, 2), 77),       # one-CTA kernel (d = 64)
])
def test_fwd_with_extra_segment_matches_oracle(B, heads, d, grid, win, shift, E):
    T, H, W = grid
    q, k, v = make_custom(B, heads, d, T, H, W, seed=E)
    kx, vx = _extra(B, E, heads, d, seed=1000 + E)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    out = sw.swattn_fwd_mem(q.to(dev), k.to(dev), v.to(dev), kx.to(dev), vx.to(dev), grid, win, shift, scale)
    assert sw.last_device_error() == sw.BASA_OK
    ref = oracle.swattn_fwd_mem(q, k, v, kx, vx, E, B, heads, T, H, W, d, win, shift, scale)
    _check(out.float().cpu().numpy(), ref, f"extra E={E} grid={grid} win={win} d={d}")


def test_fwd_with_empty_extra_segment_is_bitwise_the_plain_forward():
    grid, win, shift, d = (1, 24, 24), (1, 8, 8), (0, 4, 4), 128
    q, k, v = make_custom(1, 2, d, *grid, seed=5)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    empty = torch.empty((1, 0, 2, d), dtype=torch.bfloat16, device=dev)
    a = sw.swattn_fwd_mem(qd, kd, vd, empty, empty, grid, win, shift)
    b = sw.swattn_fwd(qd, kd, vd, grid, win, shift)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("d,grid,win,shift,pool", [
    (128, (1, 32, 32), (1, 8, 8), (0, 4, 4), (1, 4, 4)),         # the pages' FLUX setting (p = 4), small grid
    (128, (3, 12, 20), (3, 6, 10), (0, 3, 5), (1, 4, 4)),        # video: full temporal extent, spatial pooling
])
def test_pooled_memory_pipeline(d, grid, win, shift, pool):
    # GPU: kv_pool then the forward with the pooled tokens; oracle: its own pooling,
    # rounded to bf16 the way every K/V operand is, then its forward
    T, H, W = grid
    B, heads = 1, 2
    q, k, v = make_custom(B, heads, d, T, H, W, seed=7)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kbar, vbar = sw.kv_pool(kd, vd, grid, pool)
    out = sw.swattn_fwd_mem(qd, kd, vd, kbar, vbar, grid, win, shift)
    assert sw.last_device_error() == sw.BASA_OK
    G = oracle.n_pooled(T, H, W, pool)
    kb = oracle.round_to_bf16_bits(oracle.kv_pool(k, B, heads, T, H, W, d, pool))
    vb = oracle.round_to_bf16_bits(oracle.kv_pool(v, B, heads, T, H, W, d, pool))
    ref = oracle.swattn_fwd_mem(q, k, v, kb, vb, G, B, heads, T, H, W, d, win, shift, 1.0 / math.sqrt(d))
    _check(out.float().cpu().numpy(), ref, f"pooled memory grid={grid} pool={pool}")


def _text_plus_memory(kd, vd, grid, pool, n_text, seed):
    """The extra segment of the FLUX-like joint attention: n_text text tokens
    (seeded N(0,1) bf16, [B, n_text, heads, d]) followed by the pooled memory
    of K and V; returns the GPU tensors and the oracle's copy of the segment
    (text bits as drawn, pooled tokens from the oracle's own pooling rounded to
    bf16)."""
    B, _, heads, d = kd.shape
    kt, vt, _ = make_custom(B, heads, d, 1, 1, n_text, seed=seed)
    kbar, vbar = sw.kv_pool(kd, vd, grid, pool)
    kx = torch.cat([kt.to(kd.device), kbar], dim=1).contiguous()
    vx = torch.cat([vt.to(kd.device), vbar], dim=1).contiguous()
    return kx, vx, kt, vt


def _oracle_segment(t, x, B, heads, grid, d, pool):
    """Text bits followed by the oracle's pooled memory of x, as uint16 bf16 bits."""
    pooled = oracle.round_to_bf16_bits(oracle.kv_pool(x, B, heads, *grid, d, pool))
    return np.ascontiguousarray(np.concatenate([oracle._bits(t), pooled], axis=1))


def test_text_and_pooled_memory_flux1024_every_element():
    # visual queries of FLUX-1024 attend to their window, 512 text tokens and the
    # 1x4x4 pooled memory (256 tokens), in one softmax
    wl = BY_NAME["flux-1024px-64x64-w16"]
    pool, n_text = (1, 4, 4), 512
    q, k, v = make_qkv(wl)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kx, vx, kt, vt = _text_plus_memory(kd, vd, wl.grid, pool, n_text, seed=4242)
    E = kx.shape[1]
    assert E == n_text + oracle.n_pooled(*wl.grid, pool)
    shift = wl.shifts[1]
    out = sw.swattn_fwd_mem(qd, kd, vd, kx, vx, wl.grid, wl.win, shift, wl.scale)
    assert sw.last_device_error() == sw.BASA_OK
    kxs = _oracle_segment(kt, k, wl.B, wl.heads, wl.grid, wl.d, pool)
    vxs = _oracle_segment(vt, v, wl.B, wl.heads, wl.grid, wl.d, pool)
    ref = oracle.swattn_fwd_mem(q, k, v, kxs, vxs, E, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, wl.scale)
    _check(out.float().cpu().numpy(), ref, "FLUX-1024 text + pooled memory")


def test_text_and_pooled_memory_flux4096_sampled():
    # the benchmark's text_memory configuration: FLUX-4096, 512 text tokens plus the
    # 1x4x4 pooled memory (4,096 tokens); sampled rows, one whole window included
    wl = BY_NAME["flux-4096px-256x256-w32"]
    pool, n_text = (1, 4, 4), 512
    q, k, v = make_qkv(wl)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kx, vx, kt, vt = _text_plus_memory(kd, vd, wl.grid, pool, n_text, seed=4343)
    E = kx.shape[1]
    shift = wl.shifts[1]
    out = sw.swattn_fwd_mem(qd, kd, vd, kx, vx, wl.grid, wl.win, shift, wl.scale)
    assert sw.last_device_error() == sw.BASA_OK
    kxs = _oracle_segment(kt, k, wl.B, wl.heads, wl.grid, wl.d, pool)
    vxs = _oracle_segment(vt, v, wl.B, wl.heads, wl.grid, wl.d, pool)
    rng = np.random.default_rng(77)
    tri = _sample_triples(wl, shift, 600, rng)
    none = np.full((wl.B, wl.heads, sw.n_windows(wl.grid, wl.win)), -1, dtype=np.int32)
    ref = _oracle_rows_threaded(oracle.swattn_rows_route, tri, oracle._bits(q), oracle._bits(k), oracle._bits(v),
                                none, kxs, vxs, E, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, wl.scale)
    got = out[tri[:, 0], tri[:, 1], tri[:, 2]].float().cpu().numpy()
    _check(got, ref, "FLUX-4096 text + pooled memory")


# ---------------------------------------------------------------- true-window routing (§3.3)

ROUTE_TAU = 1e-4   # score margin, relative to the row's largest |s_ij|, inside which fp32 may pick either


def _check_routes(got, ref, scores, what=""):
    """The GPU's routed windows against the oracle's.  Where the oracle's best
    candidate leads the runner-up by more than the margin the two must agree;
    elsewhere (a near tie in fp64) the GPU's choice must be a candidate within
    the margin of the best.  Windows without candidates must get -1 on both."""
    got = np.asarray(got).reshape(ref.shape)
    assert np.array_equal(got == -1, ref == -1), f"{what}: candidate-less windows differ"
    cand = np.isfinite(scores)
    srt = np.sort(np.where(cand, scores, -np.inf), axis=-1)[..., ::-1]
    best, second = srt[..., 0], srt[..., 1]
    scale = np.max(np.where(cand, np.abs(scores), 0.0), axis=-1)
    tau = ROUTE_TAU * scale + 1e-12
    has = ref >= 0
    with np.errstate(invalid="ignore"):          # -inf - -inf where a window has < 2 candidates
        gap = np.where(np.isfinite(second), best - second, np.inf)
    decisive = has & (gap > tau)
    assert np.array_equal(got[decisive], ref[decisive]), f"{what}: routes differ on decisive windows"
    idx = np.clip(got, 0, None)[..., None]
    picked = np.take_along_axis(scores, idx, axis=-1)[..., 0]
    assert np.all(~has | (np.isfinite(picked) & (picked >= best - tau))), f"{what}: invalid near-tie pick"
    assert decisive.sum() >= 0.9 * has.sum(), f"{what}: too few decisive windows to be a test"
    return int(decisive.sum()), int(has.sum())


@pytest.mark.parametrize("B,heads,d,grid,win,shift,radius", [
    (2, 3, 128, (1, 24, 24), (1, 8, 8), (0, 4, 4), 1),          # image: 3x3 windows
    (1, 2, 64, (4, 17, 22), (2, 6, 5), (1, 3, 2), 1),           # temporal windows, truncated h and w
    (1, 2, 128, (3, 20, 26), (3, 5, 6), (0, 2, 3), 2),          # full temporal extent, radius 2
    (1, 2, 128, (2, 8, 8), (1, 8, 8), (1, 0, 0), 1),            # one spatial window: nothing to route
])
def test_route_matches_oracle(B, heads, d, grid, win, shift, radius):
    T, H, W = grid
    q, k, _ = make_custom(B, heads, d, T, H, W, seed=radius + d)
    got = sw.route(q.cuda(), k.cuda(), grid, win, shift, radius).cpu().numpy()
    ref, scores = oracle.route(q, k, B, heads, T, H, W, d, win, shift, radius, with_scores=True)
    _check_routes(got, ref, scores, f"grid={grid} win={win} radius={radius}")


def test_route_is_deterministic():
    grid, win, shift = (3, 20, 26), (3, 5, 6), (0, 2, 3)
    q, k, _ = make_custom(1, 4, 128, *grid, seed=3)
    qd, kd = q.cuda(), k.cuda()
    a = sw.route(qd, kd, grid, win, shift)
    for _ in range(3):
        assert torch.equal(a, sw.route(qd, kd, grid, win, shift))


def test_route_radius_beyond_the_window_grid():
    # a radius past the window grid (up to INT_MAX) selects every spatial neighbour
    grid, win, shift = (2, 20, 26), (1, 5, 6), (1, 2, 3)
    q, k, _ = make_custom(1, 2, 128, *grid, seed=31)
    qd, kd = q.cuda(), k.cuda()
    a = sw.route(qd, kd, grid, win, shift, radius=5)             # covers the 4 x 5 window grid
    for big in (6, 1000, 2 ** 31 - 1):
        assert torch.equal(a, sw.route(qd, kd, grid, win, shift, radius=big)), big
    ref, scores = oracle.route(q, k, 1, 2, *grid, 128, win, shift, 5, with_scores=True)
    _check_routes(a.cpu().numpy(), ref, scores, "radius covering the grid")


@pytest.mark.parametrize("wl", WORKLOADS[1:], ids=lambda w: w.name)
def test_route_full_size_workloads(wl):
    q, k, _ = make_qkv(wl)
    shift = wl.shifts[-1]
    got = sw.route(q.cuda(), k.cuda(), wl.grid, wl.win, shift).cpu().numpy()
    ref, scores = oracle.route(q, k, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, 1, with_scores=True)
    _check_routes(got, ref, scores, wl.name)


def _oracle_routes(q, k, B, heads, grid, d, win, shift):
    routed = oracle.route(q, k, B, heads, *grid, d, win, shift, 1)
    routed[0, 0, 0] = -1            # one window with nothing routed
    return routed


@pytest.mark.parametrize("B,heads,d,grid,win,shift,E", [
    (1, 2, 128, (1, 24, 24), (1, 8, 8), (0, 4, 4), 0),          # pair kernel, one partial routed tile
    (1, 2, 128, (2, 9, 20), (2, 9, 7), (1, 4, 3), 37),          # truncated windows routed to full ones
    (1, 2, 128, (1, 40, 40), (1, 20, 20), (0, 10, 10), 0),      # four tiles per window, ragged
    (1, 1, 128, (1, 48, 48), (1, 24, 24), (0, 0, 0), 50),       # two pair units per window, five routed tiles
    (2, 2, 64, (3, 10, 13), (2, 4, 5), (1, 3, 2), 0),           # one-CTA kernel (d = 64)
    (1, 2, 64, (2, 16, 16), (2, 8, 8), (0, 4, 4), 20),          # one-CTA kernel, full tiles plus memory
])
def test_fwd_route_matches_oracle(B, heads, d, grid, win, shift, E):
    T, H, W = grid
    q, k, v = make_custom(B, heads, d, T, H, W, seed=11 + E)
    kx, vx = _extra(B, max(E, 1), heads, d, seed=2000 + E)
    kx, vx = kx[:, :E].contiguous(), vx[:, :E].contiguous()
    routed = _oracle_routes(q, k, B, heads, grid, d, win, shift)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    rd = torch.from_numpy(routed).to(dev)
    out = sw.swattn_fwd_route(q.to(dev), k.to(dev), v.to(dev), rd, grid, win, shift,
                              kx.to(dev) if E else None, vx.to(dev) if E else None, scale)
    assert sw.last_device_error() == sw.BASA_OK
    ref = oracle.swattn_fwd_route(q, k, v, routed, kx if E else None, vx if E else None, E, B, heads, T, H, W,
                                  d, win, shift, scale)
    _check(out.float().cpu().numpy(), ref, f"routed E={E} grid={grid} win={win} d={d}")


@pytest.mark.parametrize("d", [128, 64])
def test_fwd_route_with_nothing_routed_is_bitwise_the_memory_forward(d):
    grid, win, shift = (1, 24, 24), (1, 8, 8), (0, 4, 4)
    q, k, v = make_custom(1, 2, d, *grid, seed=5)
    kx, vx = _extra(1, 9, 2, d, seed=6)
    dev = torch.device("cuda:0")
    qd, kd, vd, kxd, vxd = (t.to(dev) for t in (q, k, v, kx, vx))
    none = torch.full((1, 2, 9), -1, dtype=torch.int32, device=dev)
    a = sw.swattn_fwd_route(qd, kd, vd, none, grid, win, shift, kxd, vxd)
    b = sw.swattn_fwd_mem(qd, kd, vd, kxd, vxd, grid, win, shift)
    c = sw.swattn_fwd_route(qd, kd, vd, none, grid, win, shift)
    e = sw.swattn_fwd(qd, kd, vd, grid, win, shift)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, e)


@pytest.mark.parametrize("d,grid,win,shift,pool", [
    (128, (3, 20, 26), (3, 5, 6), (0, 2, 3), (1, 4, 4)),        # video: full temporal extent
    (128, (1, 32, 32), (1, 8, 8), (0, 4, 4), (1, 4, 4)),        # image
])
def test_full_basa_pipeline(d, grid, win, shift, pool):
    # S_i = W_i u R_i u G: GPU route, GPU pooling, GPU forward; the oracle runs its
    # own routing and pooling (rounded to bf16 like every K/V operand) and forward
    T, H, W = grid
    B, heads = 1, 2
    q, k, v = make_custom(B, heads, d, T, H, W, seed=8)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rd = sw.route(qd, kd, grid, win, shift)
    kbar, vbar = sw.kv_pool(kd, vd, grid, pool)
    out = sw.swattn_fwd_route(qd, kd, vd, rd, grid, win, shift, kbar, vbar)
    assert sw.last_device_error() == sw.BASA_OK
    routed, scores = oracle.route(q, k, B, heads, T, H, W, d, win, shift, 1, with_scores=True)
    dec, tot = _check_routes(rd.cpu().numpy(), routed, scores, "pipeline")
    assert dec == tot, "this case is chosen so that every routing decision is clear"
    G = oracle.n_pooled(T, H, W, pool)
    kb = oracle.round_to_bf16_bits(oracle.kv_pool(k, B, heads, T, H, W, d, pool))
    vb = oracle.round_to_bf16_bits(oracle.kv_pool(v, B, heads, T, H, W, d, pool))
    ref = oracle.swattn_fwd_route(q, k, v, routed, kb, vb, G, B, heads, T, H, W, d, win, shift,
                                  1.0 / math.sqrt(d))
    _check(out.float().cpu().numpy(), ref, f"full BASA grid={grid}")


@pytest.mark.parametrize("wl", [WORKLOADS[4], WORKLOADS[5]], ids=lambda w: w.name)
def test_full_basa_full_size_sampled(wl):
    # the launch configuration the benchmark's routing key times: routing, 1x4x4
    # pooled memory and the routed forward, at full size; sampled rows
    pool = (1, 4, 4)
    q, k, v = make_qkv(wl)
    shift = wl.shifts[-1]
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    routed = oracle.route(q, k, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift, 1)
    kbar, vbar = sw.kv_pool(kd, vd, wl.grid, pool)
    out = sw.swattn_fwd_route(qd, kd, vd, torch.from_numpy(routed).to(dev), wl.grid, wl.win, shift, kbar, vbar,
                              wl.scale)
    assert sw.last_device_error() == sw.BASA_OK
    G = oracle.n_pooled(*wl.grid, pool)
    kb = oracle.round_to_bf16_bits(oracle.kv_pool(k, wl.B, wl.heads, *wl.grid, wl.d, pool))
    vb = oracle.round_to_bf16_bits(oracle.kv_pool(v, wl.B, wl.heads, *wl.grid, wl.d, pool))
    rng = np.random.default_rng(wl.seed + 50)
    # random rows plus the first 300 queries of one window (three tiles, so the
    # tile seams are covered; the oracle's cost per row grows with the key count)
    tri = _sample_triples(wl, shift, 800, rng)
    tri = tri[:800 + 300]
    ref = oracle.swattn_rows_route(q, k, v, routed, kb, vb, G, wl.B, wl.heads, *wl.grid, wl.d, wl.win, shift,
                                   wl.scale, tri)
    got = out[tri[:, 0], tri[:, 1], tri[:, 2]].float().cpu().numpy()
    _check(got, ref, f"{wl.name} full BASA")
    assert torch.isfinite(out).all()
