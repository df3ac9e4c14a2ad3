"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Method: "Backend-Agnostic Sparse Attention for Fast High-Resolution Visual
Generation" (BASA), §3.1 "Shifted Window Sparse Attention" (roll by -Delta,
non-overlapping windows, softmax attention per window, roll back by +Delta),
§3.1 "Attention complexity" and Table 3 (FLOP accounting).

Each pin is chosen so that a plausible slip in the oracle fails at least one:
  * the roll direction and window numbering -> hand-worked index maps;
  * the softmax / scale / transposition     -> full-grid window equals plain
    attention, two-token closed form;
  * window membership and the un-roll        -> masked full attention built from
    numpy.roll;
  * truncated windows                         -> non-divisible grids in the
    masked comparison and in the hand-worked 3D map;
  * invariances the pages imply               -> shifts by whole windows or by
    the grid size change nothing.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from brute_force import (bf16_bits_to_f64, full_attention, masked_window_attention,
                         window_id_of_token)
from shifted_window_attention_swattn_b200.inputs import make_custom

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(B, heads, d, T, H, W, seed, dist="normal"):
    q, k, v = make_custom(B, heads, d, T, H, W, seed, dist=dist)
    bits = [oracle._bits(x) for x in (q, k, v)]
    f64 = [bf16_bits_to_f64(b).reshape(B, T * H * W, heads, d) for b in bits]
    return bits, f64


def _read_index_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "index_maps.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case"):
                kv = dict(tok.split("=") for tok in line.split()[1:])
                cur = {k: tuple(int(x) for x in v.split(",")) for k, v in kv.items()}
                cur["rows"] = []
            elif line == "end":
                cases.append(cur)
                cur = None
            else:
                cur["rows"].append([int(x) for x in line.split()])
    return cases


@pytest.mark.parametrize("case", _read_index_cases(), ids=lambda c: f"{c['grid']}-{c['shift']}")
def test_index_map_matches_hand_worked_cases(case):
    T, H, W = case["grid"]
    tos, cnt = oracle.index_map(T, H, W, case["win"], case["shift"])
    expect = np.array(case["rows"], dtype=np.int32)
    np.testing.assert_array_equal(tos, expect)
    np.testing.assert_array_equal(cnt, (expect >= 0).sum(axis=1))


def test_roll_direction_is_observable():
    # A shift that is not half the window must give a map that differs from
    # the opposite shift, so a sign slip cannot hide behind symmetric cases.
    a, _ = oracle.index_map(1, 4, 4, (1, 2, 2), (0, 1, 1))
    b, _ = oracle.index_map(1, 4, 4, (1, 2, 2), (0, -1, -1))
    assert not np.array_equal(a, b)


@pytest.mark.parametrize("grid,win,shift", [
    ((1, 6, 10), (1, 3, 4), (0, 2, 7)),
    ((3, 5, 7), (2, 2, 3), (1, 4, 5)),
    ((4, 4, 4), (4, 4, 4), (0, 0, 0)),
    ((2, 3, 9), (1, 3, 9), (1, -1, -13)),
    ((5, 1, 1), (2, 1, 1), (3, 0, 0)),
])
def test_index_map_is_bijection_consistent_with_numpy_roll(grid, win, shift):
    T, H, W = grid
    tos, cnt = oracle.index_map(T, H, W, win, shift)
    valid = tos[tos >= 0]
    assert sorted(valid.tolist()) == list(range(T * H * W))
    wid = window_id_of_token(T, H, W, win, shift)
    for m in range(tos.shape[0]):
        members = tos[m, :cnt[m]]
        assert np.all(wid[members] == m)
        assert np.all(tos[m, cnt[m]:] == -1)


@pytest.mark.parametrize("shift", [(0, 0, 0), (0, 3, 5), (1, -2, 9)])
def test_window_equal_to_grid_is_full_attention(shift):
    # Window = whole grid: the roll is a permutation and attention is
    # permutation-equivariant, so the result is plain full attention.
    B, heads, d, T, H, W = 2, 2, 16, 2, 5, 6
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=11)
    scale = 1.0 / math.sqrt(d)
    got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, (T, H, W), shift, scale)
    ref = full_attention(q, k, v, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("grid,win,shift,d", [
    ((1, 8, 8), (1, 4, 4), (0, 2, 2), 16),
    ((1, 6, 10), (1, 3, 4), (0, 2, 7), 8),        # W not divisible by w_w
    ((3, 5, 7), (2, 2, 3), (1, 4, 5), 8),         # 3D, nothing divisible
    ((3, 4, 6), (3, 2, 3), (-1, 5, -4), 8),       # negative and oversized shifts
    ((2, 3, 3), (1, 1, 1), (1, 1, 1), 4),         # one-token windows
])
def test_matches_masked_full_attention(grid, win, shift, d):
    T, H, W = grid
    B, heads = 2, 3
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=sum(grid) + d)
    scale = 0.7 / math.sqrt(d)
    got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, shift, scale)
    ref = masked_window_attention(q, k, v, T, H, W, win, shift, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_shift_by_whole_windows_is_bitwise_unshifted():
    # Windows divide the grid: a shift by whole windows only relabels windows.
    B, heads, d, T, H, W = 1, 2, 16, 2, 8, 12
    win = (1, 4, 3)
    bits, _ = _qkv(B, heads, d, T, H, W, seed=5)
    base = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, (0, 0, 0), 0.25)
    for shift in [(1, 4, 3), (0, 8, 9), (1, -4, -6)]:
        got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, shift, 0.25)
        assert np.array_equal(got, base), shift


def test_shift_by_grid_extent_is_identity():
    B, heads, d, T, H, W = 1, 1, 8, 3, 5, 7
    win = (2, 2, 3)
    bits, _ = _qkv(B, heads, d, T, H, W, seed=6)
    a = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, (1, 2, 3), 0.3)
    b = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, (1 + T, 2 - 2 * H, 3 + 5 * W), 0.3)
    assert np.array_equal(a, b)


def test_scale_zero_gives_window_mean_of_v():
    B, heads, d, T, H, W = 1, 2, 8, 2, 6, 5
    win, shift = (2, 4, 2), (1, 3, 1)
    bits, (_, _, v) = _qkv(B, heads, d, T, H, W, seed=7)
    got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, shift, 0.0)
    wid = window_id_of_token(T, H, W, win, shift)
    ref = np.empty_like(v)
    for m in np.unique(wid):
        sel = wid == m
        ref[:, sel] = v[:, sel].mean(axis=1, keepdims=True)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


def test_constant_v_gives_constant_output():
    B, heads, d, T, H, W = 1, 2, 8, 1, 6, 6
    bits, _ = _qkv(B, heads, d, T, H, W, seed=8)
    vconst = np.full_like(bits[2], 0x3FC0)   # bf16 1.5
    got = oracle.swattn_fwd(bits[0], bits[1], vconst, B, heads, T, H, W, d, (1, 3, 2), (0, 1, 1), 1.0)
    np.testing.assert_allclose(got, 1.5, rtol=0, atol=1e-14)


def test_single_token_windows_return_v_exactly():
    B, heads, d, T, H, W = 1, 2, 8, 2, 3, 4
    bits, (_, _, v) = _qkv(B, heads, d, T, H, W, seed=9)
    got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, (1, 1, 1), (1, 2, 3), 1.0)
    assert np.array_equal(got, v)


def test_two_token_window_closed_form():
    # softmax over two keys: o = (e^{s1} v1 + e^{s2} v2) / (e^{s1} + e^{s2}).
    B, heads, d, T, H, W = 1, 1, 4, 1, 1, 2
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=10)
    scale = 0.5
    got = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, (1, 1, 2), (0, 0, 1), scale)
    for i in range(2):
        s = [scale * float(np.dot(q[0, i, 0], k[0, j, 0])) for j in range(2)]
        e = [math.exp(x) for x in s]
        o = (e[0] * v[0, 0, 0] + e[1] * v[0, 1, 0]) / (e[0] + e[1])
        np.testing.assert_allclose(got[0, i, 0], o, rtol=1e-14, atol=1e-15)


def test_rows_agree_bitwise_with_full_forward():
    B, heads, d, T, H, W = 2, 3, 16, 3, 5, 7
    win, shift = (2, 2, 3), (1, -2, 4)
    bits, _ = _qkv(B, heads, d, T, H, W, seed=12)
    full = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, win, shift, 0.4)
    rng = np.random.default_rng(0)
    triples = np.stack([rng.integers(0, B, 40), rng.integers(0, T * H * W, 40),
                        rng.integers(0, heads, 40)], axis=1)
    rows = oracle.swattn_rows(*bits, B, heads, T, H, W, d, win, shift, 0.4, triples)
    for r, (b, t, h) in enumerate(triples):
        assert np.array_equal(rows[r], full[b, t, h])


def test_head_range_leaves_other_heads_untouched():
    B, heads, d, T, H, W = 1, 4, 8, 1, 4, 4
    bits, _ = _qkv(B, heads, d, T, H, W, seed=13)
    full = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, (1, 2, 2), (0, 1, 1), 0.3)
    part = oracle.swattn_fwd(*bits, B, heads, T, H, W, d, (1, 2, 2), (0, 1, 1), 0.3, head_range=(1, 3))
    assert np.array_equal(part[:, :, 1:3], full[:, :, 1:3])
    assert np.isnan(part[:, :, 0]).all() and np.isnan(part[:, :, 3]).all()


def test_rejects_bad_geometry():
    with pytest.raises(ValueError):
        oracle.index_map(1, 4, 4, (1, 5, 2), (0, 0, 0))
    with pytest.raises(ValueError):
        oracle.index_map(1, 4, 4, (0, 2, 2), (0, 0, 0))


def _read_flop_rows():
    rows = []
    with open(os.path.join(GOLDEN, "flop_counts.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                p = line.split()
                rows.append((p[0], float(p[1]), [int(x) for x in p[2:]]))
    return rows


@pytest.mark.parametrize("row", _read_flop_rows(), ids=lambda r: r[0])
def test_flop_metric_matches_printed_table(row):
    name, printed_tflops, (T, H, W, heads, d, wt, wh, ww, terms) = row
    local = oracle.flops(1, heads, T, H, W, d, (wt, wh, ww))
    assert abs(terms * local / 1e12 - printed_tflops) / printed_tflops < 0.01


def test_flops_closed_form_divisible_and_truncated():
    # Divisible: 4 * N * n_w * d * heads * B.
    assert oracle.flops(2, 3, 2, 8, 12, 16, (1, 4, 3)) == 4 * (2 * 8 * 12) * 12 * 16 * 3 * 2
    # Truncated: sum over windows of 4 n_m^2 d; W = 5 cut into 2 + 2 + 1.
    assert oracle.flops(1, 1, 1, 1, 5, 8, (1, 1, 2)) == 4 * 8 * (4 + 4 + 1)


def test_masked_attention_helper_is_itself_sane():
    # The brute force must reduce to plain attention when every token shares a
    # window, and to identity when every window has one token.
    B, heads, d, T, H, W = 1, 1, 4, 1, 2, 3
    _, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=14)
    full = full_attention(q, k, v, 0.5)
    np.testing.assert_allclose(
        masked_window_attention(q, k, v, T, H, W, (T, H, W), (0, 0, 0), 0.5), full, atol=0)
    np.testing.assert_allclose(
        masked_window_attention(q, k, v, T, H, W, (1, 1, 1), (0, 1, 2), 0.5), v, atol=0)


# ---------------------------------------------------------------- shift schedule
# §3.1 "Interleaved shift schedule": delta = max(1, floor(w/L)), a_i = (i delta) mod w,
# b = (a_0, a_K, a_1, a_{K+1}, ...), Delta_l = (b_l + c_s) mod w.  Values below are
# worked by hand from that definition.

@pytest.mark.parametrize("L,w,expected", [
    (8, 16, [0, 8, 2, 10, 4, 12, 6, 14]),     # delta 2, K 4
    (4, 16, [0, 8, 4, 12]),                   # delta 4, K 2
    (5, 7, [0, 3, 1, 4, 2]),                  # delta 1, K 3: odd L, a_{K-1} last
    (6, 4, [0, 3, 1, 0, 2, 1]),               # L > w: delta 1, a wraps mod w
    (3, 32, [0, 20, 10]),                     # delta 10, K 2
    (1, 9, [0]),
])
def test_shift_schedule_hand_worked(L, w, expected):
    sched = oracle.shift_schedule(L, (1, w, w))
    assert [s[1] for s in sched] == expected
    assert [s[2] for s in sched] == expected
    assert all(s[0] == 0 for s in sched)      # a window of one along t: only shift 0


def test_shift_schedule_two_layers_is_the_swin_alternation():
    # L = 2 gives delta = floor(w/2) and b = (0, floor(w/2)): Swin's alternating half shift
    for w in (7, 8, 13, 16, 32):
        assert oracle.shift_schedule(2, (w, w, w)) == [(0, 0, 0), (w // 2,) * 3]


def test_shift_schedule_step_offset_and_range():
    assert [s[1] for s in oracle.shift_schedule(2, (1, 16, 16), (0, 5, -3))] == [5, 13]
    assert [s[2] for s in oracle.shift_schedule(2, (1, 16, 16), (0, 5, -3))] == [13, 5]
    for L in range(1, 12):
        for w in (1, 3, 8, 15, 16):
            sched = oracle.shift_schedule(L, (w, w, w), (L, -L, 2 * L))
            assert all(0 <= x < w for s in sched for x in s)


def test_shift_schedule_is_a_permutation_of_the_offsets():
    # b reorders a: same multiset, every layer present once
    for L in range(1, 20):
        for w in (4, 13, 16, 32):
            delta = max(1, w // L)
            a = sorted((i * delta) % w for i in range(L))
            b = sorted(s[1] for s in oracle.shift_schedule(L, (1, w, 1)))
            assert a == b


def test_shift_schedule_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.shift_schedule(0, (1, 8, 8))
    with pytest.raises(ValueError):
        oracle.shift_schedule(4, (1, 0, 8))


# ---------------------------------------------------------------- pooled global memory (§3.2)

@pytest.mark.parametrize("grid,pool", [
    ((1, 8, 8), (1, 4, 4)),
    ((2, 5, 7), (1, 2, 3)),          # truncated patches on h and w
    ((3, 4, 6), (2, 4, 4)),          # temporal pooling, truncated along t and w
])
def test_kv_pool_matches_patch_means(grid, pool):
    from brute_force import pooled_means
    T, H, W = grid
    bits, (q, k, v) = _qkv(2, 3, 8, T, H, W, seed=sum(grid))
    got = oracle.kv_pool(bits[1], 2, 3, T, H, W, 8, pool)
    ref = pooled_means(k, T, H, W, pool)
    assert got.shape == ref.shape == (2, oracle.n_pooled(T, H, W, pool), 3, 8)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


def test_kv_pool_special_cases():
    T, H, W = 2, 3, 5
    bits, (q, k, v) = _qkv(1, 2, 4, T, H, W, seed=3)
    # patches of one token: the pooled tokens are the tokens themselves, in raster order
    np.testing.assert_array_equal(oracle.kv_pool(bits[2], 1, 2, T, H, W, 4, (1, 1, 1)), v)
    # one patch covering the grid: the mean over all tokens
    np.testing.assert_allclose(oracle.kv_pool(bits[2], 1, 2, T, H, W, 4, (T, H, W))[:, 0],
                               v.mean(axis=1), rtol=0, atol=1e-15)
    # hand-worked: a 1x2x2 grid of one channel pooled 2x2 -> the mean of its four values
    x = oracle.round_to_bf16_bits(np.array([1.0, 2.0, 4.0, 8.0]).reshape(1, 4, 1, 1))
    assert oracle.kv_pool(x, 1, 1, 1, 2, 2, 1, (1, 2, 2))[0, 0, 0, 0] == 3.75


@pytest.mark.parametrize("grid,win,shift,E", [
    ((1, 8, 8), (1, 4, 4), (0, 2, 2), 5),
    ((2, 5, 7), (1, 3, 4), (1, 4, 6), 9),        # 3D, truncated windows
    ((1, 6, 6), (1, 6, 6), (0, 0, 0), 3),        # one window: full attention plus the extra keys
])
def test_fwd_with_extra_segment_matches_masked_attention(grid, win, shift, E):
    from brute_force import masked_window_attention_with_extra
    T, H, W = grid
    B, heads, d = 2, 2, 8
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=E)
    xbits, (kx, vx, _) = _qkv(B, heads, d, 1, 1, E, seed=100 + E)
    scale = 0.6 / math.sqrt(d)
    got = oracle.swattn_fwd_mem(*bits, xbits[0], xbits[1], E, B, heads, T, H, W, d, win, shift, scale)
    ref = masked_window_attention_with_extra(q, k, v, kx, vx, T, H, W, win, shift, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_fwd_with_empty_extra_segment_is_the_plain_forward():
    T, H, W = 1, 6, 8
    bits, _ = _qkv(1, 2, 8, T, H, W, seed=4)
    empty = np.zeros(0, dtype=np.uint16)
    a = oracle.swattn_fwd_mem(*bits, empty, empty, 0, 1, 2, T, H, W, 8, (1, 3, 4), (0, 1, 2), 0.3)
    b = oracle.swattn_fwd(*bits, 1, 2, T, H, W, 8, (1, 3, 4), (0, 1, 2), 0.3)
    np.testing.assert_array_equal(a, b)


def test_fwd_with_extra_segment_of_one_dominant_key():
    # an extra key whose logit dominates every window key turns every output row into its value
    T, H, W, d = 1, 4, 4, 4
    bits, (q, k, v) = _qkv(1, 1, d, T, H, W, seed=9, dist="uniform")
    qf = np.ones((1, T * H * W, 1, d))
    qb = oracle.round_to_bf16_bits(qf)
    kx = oracle.round_to_bf16_bits(np.full((1, 1, 1, d), 64.0))
    vx = oracle.round_to_bf16_bits(np.arange(d, dtype=np.float64).reshape(1, 1, 1, d))
    out = oracle.swattn_fwd_mem(qb, bits[1], bits[2], kx, vx, 1, 1, 1, T, H, W, d,
                                (1, 2, 2), (0, 1, 1), 1.0)
    np.testing.assert_allclose(out[0, :, 0, :], np.tile(np.arange(d), (T * H * W, 1)), rtol=0, atol=1e-30)


# ---------------------------------------------------------------- §3.3 true-window routing

@pytest.mark.parametrize("grid,win,shift,radius", [
    ((1, 12, 12), (1, 4, 4), (0, 0, 0), 1),
    ((1, 11, 13), (1, 4, 5), (0, 3, 7), 1),      # truncated windows, shifted partition
    ((4, 9, 10), (2, 3, 4), (1, 2, 6), 1),       # temporal windows: candidates share m_t
    ((3, 9, 10), (3, 3, 4), (0, 1, 2), 2),       # full temporal extent, radius 2
])
def test_route_matches_numpy_restatement(grid, win, shift, radius):
    from brute_force import routed_windows
    T, H, W = grid
    B, heads, d = 2, 3, 8
    bits, (q, k, _) = _qkv(B, heads, d, T, H, W, seed=sum(grid) + radius)
    got, got_s = oracle.route(bits[0], bits[1], B, heads, T, H, W, d, win, shift, radius, with_scores=True)
    ref, ref_s = routed_windows(q, k, T, H, W, win, shift, radius)
    np.testing.assert_allclose(got_s, ref_s, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(got, ref)


def test_route_candidates_are_spatial_neighbours():
    T, H, W, win = 4, 12, 15, (2, 3, 3)
    bits, _ = _qkv(1, 2, 8, T, H, W, seed=21)
    routed = oracle.route(bits[0], bits[1], 1, 2, T, H, W, 8, win, (1, 1, 2), 1)
    nwin = (2, 4, 5)
    for h in range(2):
        for i in range(40):
            r = int(routed[0, h, i])
            ti, hi, wi = np.unravel_index(i, nwin)
            tr, hr, wr = np.unravel_index(r, nwin)
            assert r != i and tr == ti and abs(hr - hi) <= 1 and abs(wr - wi) <= 1


def test_route_planted_pair_and_tie_rule():
    # window 5 of a 4x4 window grid gets query mean e_0 * 2; only window 10's keys
    # have a component along e_0 (mean 3), so 5 routes to 10 with s = 2*3/sqrt(d);
    # every other score is exactly 0 and the lowest candidate index wins the tie
    T, H, W, d, win = 1, 8, 8, 4, (1, 2, 2)
    wid = np.arange(64).reshape(8, 8)
    wid = (wid // 8 // 2) * 4 + (wid % 8) // 2
    q = np.zeros((1, 64, 1, d)); k = np.zeros((1, 64, 1, d))
    q[0, wid.reshape(-1) == 5, 0, 0] = 2.0
    k[0, wid.reshape(-1) == 10, 0, 0] = 3.0
    routed, s = oracle.route(oracle.round_to_bf16_bits(q), oracle.round_to_bf16_bits(k), 1, 1, T, H, W, d,
                             win, (0, 0, 0), 1, with_scores=True)
    assert routed[0, 0, 5] == 10 and s[0, 0, 5, 10] == 2.0 * 3.0 / 2.0
    expected_ties = {0: 1, 3: 2, 12: 8, 15: 10, 10: 5, 6: 1}
    for i, r in expected_ties.items():
        assert routed[0, 0, i] == r, (i, routed[0, 0, i])


def test_route_degenerate_cases():
    bits, _ = _qkv(1, 2, 8, 2, 6, 6, seed=3)
    # one window per temporal slice: no candidate
    assert (oracle.route(bits[0], bits[1], 1, 2, 2, 6, 6, 8, (1, 6, 6), (0, 0, 0), 1) == -1).all()
    # radius 0: no candidate
    assert (oracle.route(bits[0], bits[1], 1, 2, 2, 6, 6, 8, (1, 2, 3), (0, 1, 1), 0) == -1).all()
    # a radius covering the grid: the argmax over every other window of the slice
    from brute_force import routed_windows
    _, (q, k, _) = _qkv(1, 2, 8, 2, 6, 6, seed=3)
    got = oracle.route(bits[0], bits[1], 1, 2, 2, 6, 6, 8, (1, 2, 3), (0, 1, 1), 9)
    _, sc = routed_windows(q, k, 2, 6, 6, (1, 2, 3), (0, 1, 1), 9)
    nW = 12
    for i in range(nW):
        same_t = [j for j in range(nW) if j // 6 == i // 6 and j != i]
        assert got[0, 0, i] == same_t[int(np.argmax(sc[0, 0, i, same_t]))]


@pytest.mark.parametrize("grid,win,shift,E", [
    ((1, 12, 12), (1, 4, 4), (0, 2, 2), 0),
    ((1, 11, 13), (1, 4, 5), (0, 3, 7), 6),      # truncated windows routed to each other
    ((3, 7, 9), (3, 3, 4), (0, 1, 2), 4),        # full temporal extent
])
def test_fwd_route_matches_masked_attention(grid, win, shift, E):
    from brute_force import masked_routed_attention
    T, H, W = grid
    B, heads, d = 2, 2, 8
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=40 + E)
    xbits, (kx, vx, _) = _qkv(B, heads, d, 1, 1, max(E, 1), seed=140 + E)
    kx, vx = kx[:, :E], vx[:, :E]
    routed = oracle.route(bits[0], bits[1], B, heads, T, H, W, d, win, shift, 1)
    routed[0, 1, 0] = -1                                     # a window with nothing routed
    scale = 0.7 / math.sqrt(d)
    got = oracle.swattn_fwd_route(*bits, routed, xbits[0][: B * E * heads * d] if E else None,
                                  xbits[1][: B * E * heads * d] if E else None, E,
                                  B, heads, T, H, W, d, win, shift, scale)
    ref = masked_routed_attention(q, k, v, routed, kx, vx, T, H, W, win, shift, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_fwd_route_with_nothing_routed_is_the_memory_forward():
    T, H, W, d, E = 1, 6, 8, 8, 3
    bits, _ = _qkv(1, 2, d, T, H, W, seed=4)
    xbits, _ = _qkv(1, 2, d, 1, 1, E, seed=5)
    none = np.full((1, 2, oracle.n_windows(T, H, W, (1, 3, 4))), -1, dtype=np.int32)
    a = oracle.swattn_fwd_route(*bits, none, xbits[0], xbits[1], E, 1, 2, T, H, W, d, (1, 3, 4), (0, 1, 2), 0.3)
    b = oracle.swattn_fwd_mem(*bits, xbits[0], xbits[1], E, 1, 2, T, H, W, d, (1, 3, 4), (0, 1, 2), 0.3)
    np.testing.assert_array_equal(a, b)


def test_fwd_route_dominant_routed_key():
    # a key in the routed window whose logit dominates: every query of the routing
    # window returns that key's value; windows 1 and 2 (which neither hold that key
    # nor route to its window) do not
    T, H, W, d, win = 1, 4, 4, 4, (1, 2, 2)
    bits, (q, k, v) = _qkv(1, 1, d, T, H, W, seed=9, dist="uniform")
    qb = oracle.round_to_bf16_bits(np.ones((1, 16, 1, d)))
    kf = bf16_bits_to_f64(bits[1]).reshape(1, 16, 1, d).copy()
    kf[0, 15] = 64.0                                         # token (3,3): window 3
    vf = bf16_bits_to_f64(bits[2]).reshape(1, 16, 1, d).copy()
    vf[0, 15] = np.arange(d)
    routed = np.array([[[3, 0, 0, 1]]], dtype=np.int32)      # window 0 -> 3
    out = oracle.swattn_fwd_route(qb, oracle.round_to_bf16_bits(kf), oracle.round_to_bf16_bits(vf), routed,
                                  None, None, 0, 1, 1, T, H, W, d, win, (0, 0, 0), 1.0)
    wid = window_id_of_token(T, H, W, win, (0, 0, 0))
    np.testing.assert_allclose(out[0, wid == 0, 0, :], np.tile(np.arange(d), (4, 1)), rtol=0, atol=1e-30)
    other = (wid == 1) | (wid == 2)
    assert np.all(np.abs(out[0, other, 0, :] - np.arange(d)).max(axis=1) > 1e-3)


@pytest.mark.parametrize("E", [0, 5])
def test_rows_route_agree_bitwise_with_full_routed_forward(E):
    T, H, W, d, win, shift = 2, 7, 9, 8, (1, 3, 4), (1, 2, 5)
    B, heads = 2, 2
    bits, (q, k, _) = _qkv(B, heads, d, T, H, W, seed=77)
    xbits, _ = _qkv(B, heads, d, 1, 1, max(E, 1), seed=78)
    kx = xbits[0][: B * E * heads * d] if E else None
    vx = xbits[1][: B * E * heads * d] if E else None
    routed = oracle.route(bits[0], bits[1], B, heads, T, H, W, d, win, shift, 1)
    routed[1, 0, 3] = -1
    full = oracle.swattn_fwd_route(*bits, routed, kx, vx, E, B, heads, T, H, W, d, win, shift, 0.4)
    rng = np.random.default_rng(0)
    triples = np.stack([rng.integers(0, B, 40), rng.integers(0, T * H * W, 40), rng.integers(0, heads, 40)], 1)
    rows = oracle.swattn_rows_route(*bits, routed, kx, vx, E, B, heads, T, H, W, d, win, shift, 0.4, triples)
    np.testing.assert_array_equal(rows, full[triples[:, 0], triples[:, 1], triples[:, 2]])


def _branch(s, v):
    """Softmax attention of one branch: (O, log-sum-exp) for logits s [n, m], values v [m, d]."""
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ v, (mx + np.log(z))[:, 0]


def test_single_softmax_equals_the_lse_merge_of_branches():
    # Appendix A.1 runs the local window and the memory as separate attention calls and
    # merges them with O = (1 - g) O_a + g O_b, g = sigmoid(l_b - l_a) (l = log-sum-exp);
    # the kernels instead run one softmax over the concatenated keys.  The two agree:
    # two-way {local} | {text + memory} and three-way {local} | {text} | {memory}
    # merges, built branch by branch in numpy, reproduce the oracle's single softmax,
    # and so does {local} | {routed} | {memory} for the routed forward (§3.3).
    T, H, W, d, win, shift = 1, 8, 12, 8, (1, 4, 4), (0, 2, 1)
    B, heads, E_txt, E_mem = 1, 2, 3, 5
    bits, (q, k, v) = _qkv(B, heads, d, T, H, W, seed=31)
    xbits, (kx, vx, _) = _qkv(B, heads, d, 1, 1, E_txt + E_mem, seed=32)
    scale = 0.9 / math.sqrt(d)
    wid = window_id_of_token(T, H, W, win, shift)
    routed = oracle.route(bits[0], bits[1], B, heads, T, H, W, d, win, shift, 1)
    single = oracle.swattn_fwd_mem(*bits, xbits[0], xbits[1], E_txt + E_mem, B, heads, T, H, W, d, win, shift,
                                   scale)
    single_rt = oracle.swattn_fwd_route(*bits, routed, xbits[0], xbits[1], E_txt + E_mem, B, heads, T, H, W, d,
                                        win, shift, scale)

    def merge(parts):
        o, lse = parts[0]
        for ob, lb in parts[1:]:
            g = 1.0 / (1.0 + np.exp(-(lb - lse)))
            o = (1.0 - g)[:, None] * o + g[:, None] * ob
            lse = np.logaddexp(lse, lb)
        return o

    for h in range(heads):
        qh, kh, vh = q[0, :, h], k[0, :, h], v[0, :, h]
        s_loc = np.where(wid[:, None] == wid[None, :], scale * qh @ kh.T, -np.inf)
        local = _branch(s_loc, vh)
        txt = _branch(scale * qh @ kx[0, :E_txt, h].T, vx[0, :E_txt, h])
        mem = _branch(scale * qh @ kx[0, E_txt:, h].T, vx[0, E_txt:, h])
        both = _branch(scale * qh @ kx[0, :, h].T, vx[0, :, h])
        np.testing.assert_allclose(merge([local, both]), single[0, :, h], rtol=0, atol=1e-13)
        np.testing.assert_allclose(merge([local, txt, mem]), single[0, :, h], rtol=0, atol=1e-13)
        rt = routed[0, h][wid]
        s_rt = np.where(rt[:, None] == wid[None, :], scale * qh @ kh.T, -np.inf)
        np.testing.assert_allclose(merge([local, _branch(s_rt, vh), both]), single_rt[0, :, h], rtol=0, atol=1e-13)
