"""Seeded synthetic workloads for shifted-window attention.

This module holds only shapes and random-number draws; it contains none of the
method's arithmetic, so both the CUDA path and the CPU oracle may be fed from
it.  The shapes stand in for DiT visual-token activations of FLUX-like images
and Wan-like videos ("Backend-Agnostic Sparse Attention for Fast
High-Resolution Visual Generation", §4.1 "Experimental Settings" and Tables 2-3
describe the pages' own FLUX.1-dev and Wan2.1 workloads; the datasets, prompts
and model weights behind them are not used).

Recipe (every workload):
  * Q, K, V drawn i.i.d. N(0, 1) in fp32 from one torch.Generator seeded with
    the workload's seed, in the order Q, K, V, then rounded to bf16;
  * layout [B, T*H*W, heads, d], raster token order (t, h, w);
  * scale = 1/sqrt(d);
  * seed = the workload's index in WORKLOADS;
  * the 4096^2 FLUX-like workload then draws one factor s_h ~ U(0.5, 2) per
    head and multiplies that head's Q and K rows by it (in fp32, before the
    bf16 rounding), so logits of head h have standard deviation s_h^2.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    win: Tuple[int, int, int]
    shifts: Tuple[Tuple[int, int, int], ...]   # the alternating per-layer shifts
    seed: int
    head_scale: bool = False                   # per-head U(0.5, 2) factor on Q and K

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_w(self) -> int:
        return self.win[0] * self.win[1] * self.win[2]

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def grid(self) -> Tuple[int, int, int]:
        return (self.T, self.H, self.W)


WORKLOADS = (
    Workload("tiny-2d-16x16-w8", 1, 2, 64, 1, 16, 16, (1, 8, 8), ((0, 0, 0), (0, 4, 4)), 0),
    Workload("flux-1024px-64x64-w16", 1, 24, 128, 1, 64, 64, (1, 16, 16),
             ((0, 0, 0), (0, 8, 8)), 1),
    Workload("flux-4096px-256x256-w32", 1, 24, 128, 1, 256, 256, (1, 32, 32),
             ((0, 0, 0), (0, 16, 16)), 2, head_scale=True),
    Workload("wan-480p-21x30x52-w7x10x13", 1, 12, 128, 21, 30, 52, (7, 10, 13),
             ((0, 0, 0), (3, 5, 6)), 3),
    Workload("wan-720p-21x45x80-w7x15x16", 1, 40, 128, 21, 45, 80, (7, 15, 16),
             ((0, 0, 0), (3, 7, 8)), 4),
    # The pages' own Wan2.1 geometry (a 1664x960, 81-frame video: latent grid
    # 21 x 60 x 104, 12 heads of 128), with the pages' spatial-only windows that
    # keep the full temporal extent: 15 x 26 (8,190 tokens) and the
    # non-divisible 10 x 10 (the last window along w holds 4 columns).
    Workload("wan-pages-21x60x104-w21x15x26", 1, 12, 128, 21, 60, 104, (21, 15, 26),
             ((0, 0, 0), (0, 7, 13)), 5),
    Workload("wan-pages-21x60x104-w21x10x10", 1, 12, 128, 21, 60, 104, (21, 10, 10),
             ((0, 0, 0), (0, 5, 5)), 6),
    # Head dimension 64 at scale (the 16x16 small case grown to a 256x256 grid
    # with 24 heads): half the MMA work per exponential of the d = 128
    # workloads, so the softmax's exponentials weigh twice as much.
    Workload("d64-256x256-w16", 1, 24, 64, 1, 256, 256, (1, 16, 16), ((0, 0, 0), (0, 8, 8)), 7),
)

BY_NAME = {w.name: w for w in WORKLOADS}


def make_qkv(wl: Workload, device="cpu", seed=None):
    """Q, K, V as bf16 [B, N, heads, d] tensors on ``device``.

    The draws are made on ``device`` by a generator of that device, so CPU and
    CUDA draws differ; callers that compare the two sides generate on the CPU
    and copy.
    """
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else int(seed))
    shape = (wl.B, wl.N, wl.heads, wl.d)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if wl.head_scale:
        s = torch.rand((wl.heads,), generator=g, device=device, dtype=torch.float32) * 1.5 + 0.5
        q.mul_(s.view(1, 1, -1, 1))
        k.mul_(s.view(1, 1, -1, 1))
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_custom(B, heads, d, T, H, W, seed, device="cpu", dist="normal"):
    """Q, K, V bf16 [B, T*H*W, heads, d] for ad-hoc test shapes."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    shape = (B, T * H * W, heads, d)
    out = []
    for _ in range(3):
        if dist == "normal":
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        elif dist == "uniform":
            x = torch.rand(shape, generator=g, device=device, dtype=torch.float32) * 2 - 1
        else:
            raise ValueError(dist)
        out.append(x.to(torch.bfloat16))
    return tuple(out)
