"""Pins for the oracle's float64 -> bfloat16 rounding (CPU only)."""

from fractions import Fraction
import math

import numpy as np
import torch

from oracle import bf16


def _exact_round_bf16(x: float) -> float:
    """Brute-force RN-even onto the bf16 grid with exact rationals (normal range only)."""
    if x == 0:
        return x
    fx = Fraction(x)
    a = abs(fx)
    e = math.floor(math.log2(a))
    # guard against log2 rounding at exact powers of two
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (e - 7)
    n = a / q
    fl = math.floor(n)
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * q
    return float(r) if fx > 0 else -float(r)


def test_matches_torch_cast_on_float32_values():
    rng = np.random.default_rng(7)
    v32 = (rng.standard_normal(300_000) * np.exp2(rng.uniform(-60, 60, 300_000))).astype(np.float32)
    ours = bf16.round_to_bf16(v32.astype(np.float64))
    th = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, th)


def test_single_rounding_from_float64():
    """Values just above a bf16 midpoint, not representable in float32: float64 must
    round up where a float32 detour would tie back to even."""
    rng = np.random.default_rng(8)
    base = torch.from_numpy(rng.standard_normal(2000).astype(np.float32)).to(torch.bfloat16)
    b = base.to(torch.float64).numpy()
    ulp = np.ldexp(1.0, np.frexp(np.abs(b))[1] - 1 - 7)
    mid_plus = b + np.sign(b) * (ulp / 2 + ulp * 2.0 ** -30)
    ours = bf16.round_to_bf16(mid_plus)
    want = np.array([_exact_round_bf16(float(x)) for x in mid_plus])
    assert np.array_equal(ours, want)
    exact_mid = b + np.sign(b) * ulp / 2
    ours_mid = bf16.round_to_bf16(exact_mid)
    want_mid = np.array([_exact_round_bf16(float(x)) for x in exact_mid])
    assert np.array_equal(ours_mid, want_mid)


def test_special_values_and_bits():
    v = np.array([0.0, -0.0, 1.0, -2.5, 3.0e38, 3.4e38, -3.4e38, np.inf], dtype=np.float64)
    r = bf16.round_to_bf16(v)
    assert r[0] == 0 and not np.signbit(r[0]) and np.signbit(r[1])
    assert r[2] == 1.0 and r[3] == -2.5
    assert np.isinf(r[5]) and r[6] == -np.inf and np.isinf(r[7])
    assert bf16.to_bits(np.array([1.0]))[0] == 0x3F80
    assert bf16.to_bits(np.array([-2.0]))[0] == 0xC000
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], dtype=np.uint16)
    assert np.array_equal(bf16.to_bits(bf16.from_bits(bits)), bits)


def test_subnormal_range():
    tiny = np.array([2.0 ** -133, 1.5 * 2.0 ** -133, 2.5 * 2.0 ** -133, 2.0 ** -127 + 2.0 ** -140])
    r = bf16.round_to_bf16(tiny)
    th = torch.from_numpy(tiny.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(r, th)
