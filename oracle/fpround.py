"""IEEE-754 rounding helpers for the oracle (test infrastructure only).

Everything works on float64 numpy arrays that hold values of the narrower
format.  Conversions use round-to-nearest, ties-to-even (RNE), the IEEE default
and the rounding the codec is specified with.

Double rounding: for +, -, *, / and sqrt of two float32 operands, computing in
float64 and then rounding to float32 gives the correctly rounded float32 result
(Figueroa 1995: a format with p' >= 2p + 2 significand bits makes the second
rounding innocuous; 53 >= 2*24 + 2).  ``fl32`` after one float64 operation is
therefore exact IEEE fp32 arithmetic.  A fused multiply-add is not covered by
that theorem, so ``fma_f32`` resolves the remaining midpoint case explicitly.
"""
import numpy as np

F16_MAX = 65504.0


def fl32(a):
    """Round to the nearest float32 (RNE) and return it as float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def fl16(a):
    """Round a float32-representable value to the nearest fp16 (RNE), as float64.

    Values beyond the fp16 range become +-inf, as IEEE conversion does; callers
    that saturate clamp before calling.
    """
    a32 = np.asarray(a, dtype=np.float64).astype(np.float32)
    with np.errstate(over="ignore"):
        return a32.astype(np.float16).astype(np.float64)


def f16_bits(a):
    """fp16 bit pattern (uint16) of an fp16-representable value."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def f16_from_bits(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def fl_bf16(a):
    """Round a float32 value to the nearest bfloat16 (RNE), as float64.

    bf16 keeps the top 16 bits of the float32 encoding.  RNE adds 0x7FFF plus
    the lowest kept bit, then truncates.  Finite inputs only.
    """
    u = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def bf16_bits(a):
    """bf16 bit pattern (uint16) of a bf16-representable value."""
    u = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_from_bits(bits):
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def fma_f32(a, b, c):
    """Correctly rounded float32 fused multiply-add fl32(a*b + c), as float64.

    a, b, c hold float32 values.  The product of two 24-bit significands is
    exact in float64, so only the final addition rounds: s = fl64(p + c).  The
    TwoSum error term e (s + e == p + c exactly, Knuth) decides the single case
    where rounding s to float32 could differ from rounding p + c: s landing
    exactly on a float32 midpoint while e != 0.  No float64 value lies strictly
    between s and p + c, so in every other case both round the same way.
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    p = a * b
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    up = np.nextafter(r, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(r, np.float32(-np.inf)).astype(np.float64)
    lo = np.where(r64 > s, dn, r64)
    hi = np.where(r64 < s, up, r64)
    mid = 0.5 * (lo + hi)
    tie = (r64 != s) & (s == mid) & (e != 0)
    out = np.where(tie, np.where(e > 0, hi, lo), r64)
    return out
