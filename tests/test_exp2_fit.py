"""The kernel's FMA-pipe exp2 polynomial: its constants are the ones the fitting
script derives from the definition of 2^f, and the fit meets its error bound."""
import os
import re

import numpy as np

from shifted_window_attention_swattn_b200 import fit_exp2

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "shifted_window_attention_swattn_b200", "csrc", "softmax_sm100.cuh")


def _kernel_constants():
    text = open(HDR).read()
    return [float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)]


def test_kernel_constants_equal_fit():
    assert _kernel_constants() == fit_exp2.coefficients_f32()


def test_fit_relative_error_below_bf16_resolution():
    err = fit_exp2.max_rel_error(_kernel_constants())
    assert err < 1e-4            # bf16 keeps 8 significant bits: 2^-8 = 3.9e-3


def test_emulated_exp2_steps_in_float32():
    # Same steps as exp2_poly2, in numpy float32: round with the magic constant,
    # polynomial on the fraction, exponent add on the bit pattern.
    c = np.array(_kernel_constants(), dtype=np.float32)
    y = np.linspace(-125.0, 8.0, 200001, dtype=np.float32)
    M = np.float32(12582912.0)
    t = (y + M).astype(np.float32)
    f = (y + (M - t)).astype(np.float32)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    bits = p.astype(np.float32).view(np.int32) + (t.view(np.int32).astype(np.int64) * 8388608).astype(np.int32)
    e = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    assert np.max(np.abs(e / ref - 1.0)) < 1.2e-4
