"""The bounded-wait error path on the GPU, without a GPU fault.

A test hook makes every launch's MMA issuer wait on an mbarrier that nothing
arrives on.  With a short wait limit the launch must give up, drain what it has
in flight, release its tensor memory, report BASA_ERR_DEVICE through
basa_swattn_last_device_error, and leave the context usable: the next launch
runs normally and matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_window_attention_swattn_b200 as sw
from shifted_window_attention_swattn_b200.inputs import make_custom

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_wait_timeout_is_reported_and_context_recovers(d):
    T, H, W, heads = 2, 16, 16, 4
    win, shift, scale = (2, 8, 8), (1, 4, 4), d ** -0.5
    q, k, v = make_custom(1, heads, d, T, H, W, 31 + d)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    assert sw.last_device_error() == sw.BASA_OK
    sw.set_wait_timeout_ns(20_000_000)
    sw.set_test_stall(True)
    try:
        sw.swattn_fwd(qd, kd, vd, (T, H, W), win, shift, scale)
        rc = sw.last_device_error()
    finally:
        sw.set_test_stall(False)
        sw.set_wait_timeout_ns(1_000_000_000)
    assert rc == sw.BASA_ERR_DEVICE
    assert sw.last_device_error() == sw.BASA_OK          # the record was cleared
    out = sw.swattn_fwd(qd, kd, vd, (T, H, W), win, shift, scale)
    assert sw.last_device_error() == sw.BASA_OK
    ref = oracle.swattn_fwd(q, k, v, 1, heads, T, H, W, d, win, shift, scale)
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() <= 2e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3
    torch.cuda.synchronize()
