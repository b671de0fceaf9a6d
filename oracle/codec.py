"""Encode / decode of a whole KV cache (test infrastructure only).

Codec-Gauge, Figure 1 and Backend compatibility: at inference the cache keys
and values are mapped into the gauge coordinates before compression or
quantization and mapped back (G^T) before attention; the backend's coding rules
and bit budget are unchanged.

Buffers (per the C library's contract):
  kv     [L, 2, B, H, T, d]      bf16 values
  G      [L, 2, H, R, g, g]      fp32 values
  block-uniform:  codes [L, 2, B, H, T/tb, d/w, tb*w*b/8]   uint8
                  z, s  [L, 2, B, H, T/tb, d/w]             fp16
  KIVI-style:     keys   codes [L, B, H, T/kt, d, kt*b/8], z, s [L, B, H, T/kt, d]
                  values codes [L, B, H, T, d/vc, vc*b/8], z, s [L, B, H, T, d/vc]
                  (stored as the s = 0 and s = 1 halves of [L, 2, B, H, ...]; both
                  halves have T*d*b/8 bytes and T*d/32 scale entries per head when
                  kt = vc = 32)
Only tokens [t0, t0 + nt) are processed (rolling append).
"""
import numpy as np

from . import gauge as _g
from . import quant as _q
from .fpround import fl32


def gauged_values(kv, G32, full_head_bf16):
    """Values the quantizer sees.

    g < d : the fp32 FMA chain of ``gauge.apply_gauge_f32_chain`` (exact).
    g == d with ``full_head_bf16``: the tensor-core contraction with G rounded
    to bf16; the oracle gives its exact value fl32(G_bf16 x) and the device's
    fp32 accumulation is compared to it within a tolerance.
    """
    if full_head_bf16:
        return _g.apply_gauge(kv, _g.round_gauge_bf16(G32))
    return _g.apply_gauge_f32_chain(kv, G32)


def encode_block_uniform(kv, G32, bits, tb=16, w=None, t0=0, nt=None, full_head_bf16=False):
    """Returns dict(codes, z, s, q, y) for tokens [t0, t0+nt)."""
    kv = np.asarray(kv, dtype=np.float64)
    g = G32.shape[-1]
    w = g if w is None else w
    T = kv.shape[-2]
    nt = T - t0 if nt is None else nt
    x = kv[..., t0:t0 + nt, :]
    y = gauged_values(x, G32, full_head_bf16)
    y = fl32(y)
    yr = _q.block_uniform_view(y, tb, w)
    q, z, s = _q.quantize_ranges(yr, bits)
    return dict(codes=_q.pack_codes(q, bits), z=z, s=s, q=q, y=y)


def decode_block_uniform(codes, z, s, G, bits, tb=16, w=None, full_head_bf16=False):
    """x_hat = G^T (s q + z) in fp64 for the encoded token range."""
    g = G.shape[-1]
    w = g if w is None else w
    q = _q.unpack_codes(codes, bits, tb * w)
    yhat = _q.dequantize(q, z[..., None], s[..., None])
    y = _q.block_uniform_unview(yhat, tb, w)
    Gd = _g.round_gauge_bf16(G) if full_head_bf16 else np.asarray(G, np.float64)
    return _g.apply_inverse_gauge(y, Gd)


def encode_kivi(kv, G32, bits, kt=32, vc=32, t0=0, nt=None):
    """KIVI-style: keys per (channel, kt tokens), values per (token, vc channels)."""
    kv = np.asarray(kv, dtype=np.float64)
    T = kv.shape[-2]
    nt = T - t0 if nt is None else nt
    y = fl32(_g.apply_gauge_f32_chain(kv[..., t0:t0 + nt, :], G32))
    qk, zk, sk = _q.quantize_ranges(_q.kivi_key_view(y[:, 0], kt), bits)
    qv, zv, sv = _q.quantize_ranges(_q.kivi_value_view(y[:, 1], vc), bits)
    return dict(key=dict(codes=_q.pack_codes(qk, bits), z=zk, s=sk, q=qk),
                value=dict(codes=_q.pack_codes(qv, bits), z=zv, s=sv, q=qv), y=y)


def decode_kivi(enc, G, bits, kt=32, vc=32):
    """Reconstruct [L, 2, B, H, nt, d] in fp64 from encode_kivi's output."""
    k, v = enc["key"], enc["value"]
    qk = _q.unpack_codes(k["codes"], bits, kt)
    qv = _q.unpack_codes(v["codes"], bits, vc)
    yk = _q.kivi_key_unview(_q.dequantize(qk, k["z"][..., None], k["s"][..., None]))
    yv = _q.kivi_value_unview(_q.dequantize(qv, v["z"][..., None], v["s"][..., None]))
    y = np.stack([yk, yv], axis=1)
    return _g.apply_inverse_gauge(y, np.asarray(G, np.float64))


def sizes(L, B, H, T, d, bits, mode="block_uniform", tb=16, w=16, kt=32, vc=32):
    """(code_bytes, scale_count) of a whole cache; s and z each hold scale_count fp16."""
    n = L * 2 * B * H * T * d
    code_bytes = n * bits // 8
    if mode == "block_uniform":
        scale_count = L * 2 * B * H * (T // tb) * (d // w)
    else:
        scale_count = L * B * H * (T // kt) * d + L * B * H * T * (d // vc)
    return code_bytes, scale_count
