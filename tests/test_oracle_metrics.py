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
