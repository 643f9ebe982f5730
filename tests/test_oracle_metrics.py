"""Pins for the oracle's metrics (CPU only)."""

import numpy as np

from oracle import metrics


def test_rel_l2_hand_values():
    assert metrics.rel_l2([3.0, 4.0], [3.0, 4.0]) == 0.0
    assert metrics.rel_l2([3.0, 4.0 + 0.5], [3.0, 4.0]) == 0.5 / 5.0
    assert metrics.rel_l2([0.0], [0.0]) == 0.0


def test_error_ratio_hand_values():
    r = np.array([1.0, 2.0, 3.0, 4.0])
    y = np.array([1.0, 2.5, 3.0, 4.01])
    assert metrics.error_ratio(y, r, atol=0.0, rtol=0.01) == 0.25


def test_bf16_ulp():
    assert metrics.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert metrics.bf16_ulp(np.array([1.99]))[0] == 2.0 ** -7
    assert metrics.bf16_ulp(np.array([-2.0]))[0] == 2.0 ** -6
    assert metrics.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133


def test_bf16_ulp_is_the_grid_spacing():
    # Against the bfloat16 grid itself: for random magnitudes across many binades, the
    # gap between a bf16 value and the next one up (torch's bf16 bit pattern + 1) is
    # the ulp the oracle reports at that value.
    import torch
    rng = np.random.default_rng(7)
    v = np.ldexp(rng.uniform(1.0, 2.0, 2000), rng.integers(-120, 120, 2000))
    b = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    bits = b.view(torch.int16)
    nxt = (bits + 1).view(torch.bfloat16)
    gap = (nxt.double() - b.double()).numpy()
    np.testing.assert_array_equal(metrics.bf16_ulp(b.double().numpy()), gap)


def test_error_ratio_boundary_is_not_an_error():
    # An output exactly on atol + rtol*|r| is inside the tolerance; just above is outside.
    r = np.array([2.0, 2.0])
    y = np.array([2.0 + 0.25 + 0.5, 2.0 + 0.25 + 0.5 + 2.0 ** -40])
    assert metrics.error_ratio(y, r, atol=0.25, rtol=0.25) == 0.5
    assert metrics.error_ratio(np.zeros(0), np.zeros(0), atol=0.0, rtol=0.0) == 0.0
