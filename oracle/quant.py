"""Fixed-rate min/max quantizers and bit packing (test infrastructure only).

Codec-Gauge, Experimental setup (backends): the block-uniform backend uses one
value range per T_b x d block and the KIVI-style backend per-channel ranges for
keys and per-token ranges for values (Liu et al. 2024c); both run at the same
bit settings (2, 3, 4, 6, 8 bits/value; 3, 4, 6 in the main results).  The
pages print no quantizer formula.  This module takes the plainest asymmetric
min/max reading, with every floating-point step an IEEE fp32 operation in RNE:

  mn, mx = min(y), max(y) over the range block            (exact; a zero
                                                            extreme is +0)
  z      = fp16_rne(clamp(mn, +-65504))                     zero point (offset)
  s      = fp16_rne(min(fl32(fl32(mx - mn) / (2^b - 1)), 65504))   step
  s == 0 -> every code is 0
  else   inv = fl32(1 / s);  t = fl32(fl32(y - z) * inv)
         q   = clamp(rne(t), 0, 2^b - 1)                    (ties to even)
  dequantized value = s * q + z

Packing: inside a range block element i (in the block's stated order) holds
bits [i*b, i*b + b) of a little-endian bit stream: stream bit k is bit (k mod 8)
of byte k // 8.  Blocks are stored back to back.
"""
import numpy as np

from .fpround import fl16, fl32, F16_MAX


def quant_params(mn, mx, bits):
    """fp16 zero point z and step s of a range block, returned as float64.

    The range ends are real numbers: -0 and +0 are the same value, so a zero
    minimum or maximum is taken as +0 (adding +0 maps -0 to +0 and leaves
    every other value unchanged), and the stored zero point of a block whose
    minimum is zero is the fp16 +0.
    """
    qmax = float(2 ** bits - 1)
    mn = np.asarray(mn, dtype=np.float64) + 0.0
    mx = np.asarray(mx, dtype=np.float64) + 0.0
    z = fl16(np.clip(mn, -F16_MAX, F16_MAX))
    rng = fl32(mx - mn)
    s32 = fl32(rng / qmax)
    s = fl16(np.minimum(s32, F16_MAX))
    return z, s


def quantize(y, z, s, bits):
    """Integer codes of fp32 values y against per-value z and s (broadcast)."""
    qmax = 2 ** bits - 1
    y = np.asarray(y, dtype=np.float64)
    z = np.broadcast_to(np.asarray(z, dtype=np.float64), y.shape)
    s = np.broadcast_to(np.asarray(s, dtype=np.float64), y.shape)
    nz = s != 0
    inv = fl32(1.0 / np.where(nz, s, 1.0))
    t = fl32(fl32(y - z) * inv)
    q = np.clip(np.rint(t), 0, qmax)
    return np.where(nz, q, 0).astype(np.int64)


def dequantize(q, z, s):
    """s * q + z in fp64 (the exact dequantized value)."""
    return np.asarray(s, np.float64) * np.asarray(q, np.float64) + np.asarray(z, np.float64)


def pack_codes(q, bits):
    """Pack codes along the last axis (n codes, n*bits % 8 == 0) into bytes."""
    q = np.asarray(q, dtype=np.int64)
    n = q.shape[-1]
    assert (n * bits) % 8 == 0
    shifts = np.arange(bits, dtype=np.int64)
    bitplanes = ((q[..., :, None] >> shifts) & 1).astype(np.uint8)   # [..., n, bits], LSB first
    stream = bitplanes.reshape(q.shape[:-1] + (n * bits,))
    return np.packbits(stream, axis=-1, bitorder="little")


def unpack_codes(packed, bits, n):
    """Inverse of pack_codes: n codes from the last axis of ``packed``."""
    packed = np.asarray(packed, dtype=np.uint8)
    stream = np.unpackbits(packed, axis=-1, bitorder="little")[..., : n * bits]
    planes = stream.reshape(packed.shape[:-1] + (n, bits)).astype(np.int64)
    return (planes << np.arange(bits, dtype=np.int64)).sum(axis=-1)


def quantize_ranges(y_ranges, bits):
    """Quantize values grouped as [..., n] (one range per leading index).

    Returns (codes [..., n], z [...], s [...]).
    """
    y_ranges = np.asarray(y_ranges, dtype=np.float64)
    z, s = quant_params(y_ranges.min(axis=-1), y_ranges.max(axis=-1), bits)
    q = quantize(y_ranges, z[..., None], s[..., None], bits)
    return q, z, s


# ---- range-block views -------------------------------------------------------

def block_uniform_view(y, tb, w):
    """[..., T, d] -> [..., T/tb, d/w, tb*w], element order token-major."""
    *lead, T, d = y.shape
    v = y.reshape(tuple(lead) + (T // tb, tb, d // w, w))
    v = np.moveaxis(v, -3, -2)                    # [..., T/tb, d/w, tb, w]
    return v.reshape(tuple(lead) + (T // tb, d // w, tb * w))


def block_uniform_unview(v, tb, w):
    *lead, nt, nw, _ = v.shape
    v = v.reshape(tuple(lead) + (nt, nw, tb, w))
    v = np.moveaxis(v, -2, -3)                    # [..., nt, tb, nw, w]
    return v.reshape(tuple(lead) + (nt * tb, nw * w))


def kivi_key_view(y, kt):
    """Keys [..., T, d] -> [..., T/kt, d, kt]: one range per channel and kt tokens."""
    *lead, T, d = y.shape
    v = y.reshape(tuple(lead) + (T // kt, kt, d))
    return np.swapaxes(v, -1, -2)


def kivi_key_unview(v):
    *lead, ng, d, kt = v.shape
    return np.swapaxes(v, -1, -2).reshape(tuple(lead) + (ng * kt, d))


def kivi_value_view(y, vc):
    """Values [..., T, d] -> [..., T, d/vc, vc]: one range per token and vc channels."""
    *lead, T, d = y.shape
    return y.reshape(tuple(lead) + (T, d // vc, vc))


def kivi_value_unview(v):
    *lead, T, ng, vc = v.shape
    return v.reshape(tuple(lead) + (T, ng * vc))
