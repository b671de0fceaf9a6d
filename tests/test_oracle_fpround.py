"""Pins of the oracle's rounding helpers against exact rational arithmetic
and against library conversions (torch's fp16 / bf16 casts)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.fpround import fl16, fl_bf16, fl32, fma_f32


def _round_f32_exact(v: Fraction) -> float:
    """Correct RNE rounding of an exact rational to float32, by brute force."""
    r = np.float32(float(v))
    cands = [np.nextafter(r, np.float32(-np.inf)), r, np.nextafter(r, np.float32(np.inf))]
    best = None
    for c in cands:
        dist = abs(Fraction(float(c)) - v)
        key = (dist, int(np.array(c, np.float32).view(np.uint32)) & 1)  # tie -> even significand
        if best is None or key < best[0]:
            best = (key, float(c))
    return best[1]


def _fma_exact(a, b, c):
    return _round_f32_exact(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def test_fma_f32_random_against_rationals():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(3000).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 30, 3000).astype(np.float32)
    b = rng.standard_normal(3000).astype(np.float32)
    c = rng.standard_normal(3000).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 30, 3000).astype(np.float32)
    got = fma_f32(a, b, c)
    want = np.array([_fma_exact(x, y, z) for x, y, z in zip(a, b, c)])
    assert np.array_equal(got, want)


def test_fma_f32_double_rounding_traps():
    # a*b = 64 - 2^-30 exactly; c = 2^30 + 128.  fl64(a*b + c) = 2^30 + 192 is a
    # float32 midpoint, so naive double rounding ties to even (2^30 + 256) while
    # the exact sum lies below it: the correct fp32 FMA gives 2^30 + 128.
    a = np.float32(64.0 * (1 + 2.0 ** -18))
    b = np.float32(1 - 2.0 ** -18)
    c = np.float32(2.0 ** 30 + 128)
    assert float(fma_f32(a, b, c)) == 2.0 ** 30 + 128
    assert float(np.float32(float(a) * float(b) + float(c))) == 2.0 ** 30 + 256  # the trap is real
    assert float(fma_f32(-a, b, -c)) == -(2.0 ** 30 + 128)  # error term of the other sign
    for x, y, z in [(a, b, c), (-a, b, -c)]:
        assert float(fma_f32(x, y, z)) == _fma_exact(x, y, z)


def test_fma_f32_signed_zero():
    z = fma_f32(np.float32(-1.0), np.float32(0.0), np.float32(0.0))
    assert float(z) == 0.0 and not np.signbit(z)
    z = fma_f32(np.float32(-1.0), np.float32(0.0), np.float32(-0.0))
    assert np.signbit(z)


def test_fl32_matches_torch_cast():
    x = np.random.default_rng(2).standard_normal(10000) * 1e3
    assert np.array_equal(fl32(x), torch.from_numpy(x).float().double().numpy())


def test_fl16_matches_torch_half_cast():
    x = (np.random.default_rng(3).standard_normal(10000) * 100).astype(np.float32)
    x[:4] = [1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -25, 3 * 2 ** -26]  # ties and subnormal ties
    assert np.array_equal(fl16(x), torch.from_numpy(x).half().double().numpy())


def test_fl_bf16_matches_torch_bfloat16_cast():
    x = (np.random.default_rng(4).standard_normal(10000) * 10).astype(np.float32)
    x[:2] = [1 + 2 ** -8, 1 + 3 * 2 ** -8]
    assert np.array_equal(fl_bf16(x), torch.from_numpy(x).bfloat16().double().numpy())
