"""Pins for the oracle's block quantisers (CPU only)."""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import e4m3, quant
from fp8_block_scaled_a8w8_b200 import inputs


def _x(M, K, seed, outliers=False):
    return inputs.activation_bf16(M, K, seed, outliers).float().numpy()


def test_hand_group_single_value():
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 37] = 3.0
    q, s = quant.quant_act_per_token_group(x)
    assert s[0, 0] == np.float32(3.0) / np.float32(448.0)
    assert q[0, 37] == 0x7E
    assert np.all(np.delete(q[0], 37) == 0)
    x[0, 37] = -3.0
    q, s = quant.quant_act_per_token_group(x)
    assert q[0, 37] == 0xFE


def test_hand_group_two_values():
    # amax 448 -> scale 1 exactly, so codes are the plain e4m3 rounding of x
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 0] = 448.0
    x[0, 1] = 1.0625  # midpoint of 1.0 and 1.125 -> even code 0x38 (1.0)
    x[0, 2] = 1.1875  # midpoint of 1.125 and 1.25 -> even code 0x3A (1.25)
    x[0, 3] = -0.0
    q, s = quant.quant_act_per_token_group(x)
    assert s[0, 0] == 1.0
    assert list(q[0, :4]) == [0x7E, 0x38, 0x3A, 0x80]


def test_per_element_scalar_restatement():
    """Element by element with numpy float32 scalars and ml_dtypes' encoder."""
    x = _x(3, 256, 11)
    q, s = quant.quant_act_per_token_group(x)
    for m in range(3):
        for g in range(2):
            blk = x[m, g * 128:(g + 1) * 128]
            amax = np.float32(0)
            for v in blk:
                amax = max(amax, np.float32(abs(v)))
            sc = np.float32(amax / np.float32(448))
            assert s[m, g] == sc
            for j, v in enumerate(blk):
                y = np.float32(np.float32(v) / sc)
                code = np.array([y], dtype=np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
                assert q[m, g * 128 + j] == code


@pytest.mark.parametrize("outliers", [False, True])
def test_max_element_is_448_and_halfulp_reconstruction(outliers):
    x = _x(64, 1024, 5, outliers)
    q, s = quant.quant_act_per_token_group(x)
    G = x.shape[1] // 128
    for g in range(G):
        blk = x[:, g * 128:(g + 1) * 128]
        qb = q[:, g * 128:(g + 1) * 128]
        imax = np.argmax(np.abs(blk), axis=1)
        assert np.all((qb[np.arange(64), imax] & 0x7F) == 0x7E)
        y = blk.astype(np.float64) / s[:, g:g + 1].astype(np.float64)
        dec = e4m3.decode(qb)
        # half the e4m3 spacing at |y| (2^-10 below the normal range), plus float32 division slack
        _, ex = np.frexp(np.maximum(np.abs(y), 2.0 ** -6))
        half = np.ldexp(1.0, ex - 1 - 3) / 2
        assert np.all(np.abs(dec - y) <= half * (1 + 1e-6) + np.abs(y) * 2.0 ** -23)


def test_zero_group_and_signed_zero():
    x = np.zeros((2, 256), dtype=np.float32)
    x[1, :128] = -0.0
    x[1, 128] = 5.0
    q, s = quant.quant_act_per_token_group(x)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0
    assert np.all(q[0] == 0) and np.all(q[1, :128] == 0x80)
    assert q[1, 128] == 0x7E and np.all(q[1, 129:] == 0)


def test_tiny_subnormal_bf16_group():
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 0] = np.float32(torch.tensor(2.0 ** -133, dtype=torch.bfloat16).float().item())
    q, s = quant.quant_act_per_token_group(x)
    assert s[0, 0] > 0
    assert q[0, 0] == 0x7E


def test_weight_block_quant_properties():
    w = inputs.weight_f32(300, 384, 3).numpy()  # 3 row blocks, last one partial (44 rows)
    q, s = quant.quant_weight_block128(w)
    assert s.shape == (3, 3)
    for nb in range(3):
        for g in range(3):
            blk = w[nb * 128:min(300, nb * 128 + 128), g * 128:(g + 1) * 128]
            amax = np.float32(np.max(np.abs(blk)))
            assert s[nb, g] == np.float32(amax / np.float32(448))
            qb = q[nb * 128:min(300, nb * 128 + 128), g * 128:(g + 1) * 128]
            r, c = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
            assert (qb[r, c] & 0x7F) == 0x7E
            y = (blk / s[nb, g]).astype(np.float32)
            ref = y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            assert np.array_equal(qb, ref)
