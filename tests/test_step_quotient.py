"""The tensor-core encoder derives the block step s = fp16(fl32(rng / qmax)) with
fp32 operations only: q0 = fl(rng c) with c = fl(1/qmax), then one correction
with the exact residual, q = fl(fl(fma(-q0, qmax, rng)) c + q0).  Its exactness
(q == the correctly rounded quotient) was established by an exhaustive run over
all 2^31 non-negative fp32 values for qmax = 3, 7, 15, 63, 255; this test pins
the claim on a large sample (random bit patterns across every binade, the
subnormals, values just around powers of two and around multiples of qmax)
with the oracle's exact fp32 fused multiply-add.
"""
import numpy as np
import pytest

from oracle.fpround import fma_f32


def _corrected_quotient(x, qmax):
    c = np.float64(np.float32(1.0 / qmax))
    q0 = (x * c).astype(np.float32).astype(np.float64)            # fl(x c)
    r = (x - q0 * qmax).astype(np.float32).astype(np.float64)     # fl(fma(-q0, qmax, x)): exact in fp64, one rounding
    return fma_f32(r, c, q0)                                       # fl(fma(r, c, q0))


def _samples(rng):
    bits = rng.integers(0, 0x7F800000, size=400_000, dtype=np.uint64).astype(np.uint32)
    sub = np.arange(1, 4096, dtype=np.uint32)                      # smallest subnormals
    pow2 = np.array([(e << 23) + d for e in range(1, 255) for d in (-2, -1, 0, 1, 2)
                     if 0 < (e << 23) + d < 0x7F800000], dtype=np.uint32)
    x = np.concatenate([bits, sub, pow2]).view(np.float32).astype(np.float64)
    return x


@pytest.mark.parametrize("qmax", [3, 7, 15, 63, 255])
def test_corrected_fp32_quotient_is_correctly_rounded(qmax):
    rng = np.random.default_rng(qmax)
    x = _samples(rng)
    # around multiples of qmax, where the quotient is (nearly) an fp32 value
    k = rng.integers(1, 1 << 24, size=100_000).astype(np.float64)
    near = (k * qmax).astype(np.float32).astype(np.float64)
    near = np.concatenate([near, np.nextafter(near.astype(np.float32), np.float32(np.inf)).astype(np.float64),
                           np.nextafter(near.astype(np.float32), np.float32(0)).astype(np.float64)])
    x = np.concatenate([x, near])
    # correctly rounded: the exact quotient of a 24-bit value by qmax is never an
    # fp32 midpoint and stays >= 2^-26 / qmax (relative) away from one, so
    # rounding the fp64 quotient to fp32 gives it
    want = (x / qmax).astype(np.float32).astype(np.float64)
    got = _corrected_quotient(x, qmax)
    assert np.array_equal(got, want)
    assert np.array_equal(_corrected_quotient(-x, qmax), -want)    # odd symmetry


def test_naive_product_is_not_enough():
    """The correction step matters: fl(rng * fl(1/qmax)) alone misses some quotients."""
    x = _samples(np.random.default_rng(1))
    c = np.float64(np.float32(1.0 / 15))
    naive = (x * c).astype(np.float32).astype(np.float64)
    assert not np.array_equal(naive, (x / 15).astype(np.float32).astype(np.float64))
