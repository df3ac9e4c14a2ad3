"""Fits the polynomial the kernel uses for part of its exp2 evaluations.

2^y for y <= 0 is evaluated as 2^j * p(f) with j = round(y) and
f = y - j in [-1/2, 1/2].  p is the degree-3 polynomial that minimises the
maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2], found here with
Lawson's iteratively reweighted least squares (a standard route to the
minimax fit), starting from a least-squares fit on Chebyshev nodes.  Only
numpy and the definition of 2^f are used.

    python -m shifted_window_attention_swattn_b200.fit_exp2

prints the coefficients (c0..c3, float32-rounded) and the achieved maximum
relative error; the kernel's constants (csrc/softmax_sm100.cuh) must equal
them, which a test checks.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, n: int = 4001, iters: int = 400):
    f = np.cos(np.pi * (np.arange(n) + 0.5) / n) * 0.5          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative-error system
    b = np.ones_like(f)
    w = np.full(n, 1.0 / n)
    coef = None
    for _ in range(iters):
        sw = np.sqrt(w)
        coef, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ coef - b)
        w = w * err
        w = w / w.sum()
    return coef


def max_rel_error(coef, n: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, n)
    p = np.polyval(np.asarray(coef, dtype=np.float64)[::-1], f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


def coefficients_f32():
    return [float(np.float32(c)) for c in fit()]


if __name__ == "__main__":
    c = coefficients_f32()
    for i, v in enumerate(c):
        print(f"c{i} = {v!r}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c):.3e}")
