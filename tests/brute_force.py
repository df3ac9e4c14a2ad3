"""Independent numpy formulations used to pin the oracle (tiny sizes only).

Shifted-window attention is restated here in a second, differently built form:
full attention over the ORIGINAL token order with a block-diagonal mask, where
two tokens may attend to each other iff they fall into the same window after
the grid is rolled by -Delta ("Backend-Agnostic Sparse Attention for Fast
High-Resolution Visual Generation", §3.1 "Shifted Window Sparse Attention").
Window membership comes from ``numpy.roll`` of a grid of token ids, not from the
oracle's index arithmetic.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp64 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def window_id_of_token(T, H, W, win, shift) -> np.ndarray:
    """[N] window id of every original token.

    numpy.roll(ids, -Delta) puts original token (i + Delta) mod n at position i;
    position i of the rolled grid lies in window (i_t // w_t, i_h // w_h, i_w // w_w).
    """
    ids = np.arange(T * H * W).reshape(T, H, W)
    rolled = np.roll(ids, shift=(-shift[0], -shift[1], -shift[2]), axis=(0, 1, 2))
    nwin = [-(-n // w) for n, w in zip((T, H, W), win)]
    ct, ch, cw = np.meshgrid(np.arange(T) // win[0], np.arange(H) // win[1],
                             np.arange(W) // win[2], indexing="ij")
    wid_at_pos = (ct * nwin[1] + ch) * nwin[2] + cw
    out = np.empty(T * H * W, dtype=np.int64)
    out[rolled.reshape(-1)] = wid_at_pos.reshape(-1)
    return out


def full_attention(q, k, v, scale, mask=None):
    """Plain softmax attention per (b, head): q, k, v fp64 [B, N, heads, d]."""
    B, N, heads, d = q.shape
    out = np.empty_like(q)
    for b in range(B):
        for h in range(heads):
            s = scale * (q[b, :, h, :] @ k[b, :, h, :].T)
            if mask is not None:
                s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ v[b, :, h, :]
    return out


def masked_window_attention(q, k, v, T, H, W, win, shift, scale):
    """Shifted-window attention as block-diagonally masked full attention."""
    wid = window_id_of_token(T, H, W, win, shift)
    mask = wid[:, None] == wid[None, :]
    return full_attention(q, k, v, scale, mask)


def pooled_means(x, T, H, W, pool):
    """[B, G, heads, d] patch means of x (fp64 [B, N, heads, d]) over the unshifted grid,
    built with explicit numpy slicing of each patch (§3.2 "K/V-Pooled Global Memory")."""
    B, N, heads, d = x.shape
    g = x.reshape(B, T, H, W, heads, d)
    out = []
    for t0 in range(0, T, pool[0]):
        for h0 in range(0, H, pool[1]):
            for w0 in range(0, W, pool[2]):
                patch = g[:, t0:t0 + pool[0], h0:h0 + pool[1], w0:w0 + pool[2]]
                out.append(patch.reshape(B, -1, heads, d).mean(axis=1))
    return np.stack(out, axis=1)


def masked_window_attention_with_extra(q, k, v, kx, vx, T, H, W, win, shift, scale):
    """Shifted-window attention where every query may also attend to the extra
    tokens kx, vx ([B, E, heads, d]): full attention over the concatenated key set
    [K; K_x] with the block-diagonal window mask widened by E always-allowed columns."""
    E = kx.shape[1]
    wid = window_id_of_token(T, H, W, win, shift)
    mask = np.concatenate([wid[:, None] == wid[None, :],
                           np.ones((wid.size, E), dtype=bool)], axis=1)
    kk = np.concatenate([k, kx], axis=1)
    vv = np.concatenate([v, vx], axis=1)
    B, N, heads, d = q.shape
    out = np.empty_like(q)
    for b in range(B):
        for h in range(heads):
            s = scale * (q[b, :, h, :] @ kk[b, :, h, :].T)
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ vv[b, :, h, :]
    return out


def routed_windows(q, k, T, H, W, win, shift, radius):
    """Top-1 routing restated with numpy (§3.3 "Content-Adaptive True-Window
    Routing"): window means from the token -> window map of ``numpy.roll``,
    candidates = other windows with the same temporal window index within spatial
    window distance ``radius``.  Returns (routed [B, heads, nW] int, scores
    [B, heads, nW, nW] with -inf off the candidates)."""
    B, N, heads, d = q.shape
    wid = window_id_of_token(T, H, W, win, shift)
    nwin = [-(-n // w) for n, w in zip((T, H, W), win)]
    nW = nwin[0] * nwin[1] * nwin[2]
    onehot = (wid[None, :] == np.arange(nW)[:, None]).astype(np.float64)   # [nW, N]
    onehot /= onehot.sum(axis=1, keepdims=True)
    mq = np.einsum("wn,bnhd->bhwd", onehot, q)
    mk = np.einsum("wn,bnhd->bhwd", onehot, k)
    ct, ch, cw = np.unravel_index(np.arange(nW), nwin)
    cand = ((ct[:, None] == ct[None, :]) & (np.abs(ch[:, None] - ch[None, :]) <= radius) &
            (np.abs(cw[:, None] - cw[None, :]) <= radius) & ~np.eye(nW, dtype=bool))
    scores = np.einsum("bhid,bhjd->bhij", mq, mk) / np.sqrt(d)
    scores = np.where(cand[None, None], scores, -np.inf)
    routed = np.where(cand.any(axis=1)[None, None], scores.argmax(axis=3), -1)
    return routed, scores


def masked_routed_attention(q, k, v, routed, kx, vx, T, H, W, win, shift, scale):
    """Full attention over [K; K_x] where a query of window i may attend to the
    keys of window i, of window routed[b, h, i] and to every extra token: the
    source S_i = W_i u R_i u G of §3.3 as a mask over the original token order."""
    B, N, heads, d = q.shape
    E = kx.shape[1]
    wid = window_id_of_token(T, H, W, win, shift)
    kk = np.concatenate([k, kx], axis=1)
    vv = np.concatenate([v, vx], axis=1)
    out = np.empty_like(q)
    for b in range(B):
        for h in range(heads):
            rt = np.asarray(routed)[b, h][wid]                       # routed window of each query
            mask = (wid[:, None] == wid[None, :]) | (rt[:, None] == wid[None, :])
            mask = np.concatenate([mask, np.ones((N, E), dtype=bool)], axis=1)
            s = scale * (q[b, :, h, :] @ kk[b, :, h, :].T)
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ vv[b, :, h, :]
    return out
