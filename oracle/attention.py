"""Decode-step attention over a decoded cache (test infrastructure only).

Codec-Gauge, Figure 1 / Backend compatibility: cached keys and values are
decoded and mapped back with G^T before standard softmax attention, which the
gauge leaves unchanged.  For a query q of head j (KV head h = j // (Hq / H),
grouped-query attention) and cached tokens t < n:
    out = sum_t softmax_t(scale q . k_t) v_t
with k_t, v_t the oracle's fp64 decode (G^T (s q + z)).
"""
import numpy as np

from . import codec as _codec


def softmax_attention(q, k, v, scale):
    """q [..., Hq, d], k and v [..., H, n, d] (H divides Hq) -> [..., Hq, d], fp64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Hq, H = q.shape[-2], k.shape[-3]
    kk = np.repeat(k, Hq // H, axis=-3)
    vv = np.repeat(v, Hq // H, axis=-3)
    s = np.einsum("...hd,...htd->...ht", q, kk) * scale
    s = s - s.max(axis=-1, keepdims=True)
    w = np.exp(s)
    w = w / w.sum(axis=-1, keepdims=True)
    return np.einsum("...ht,...htd->...hd", w, vv)


def decode_attention(q, codes, z, s, G, bits, n_tokens, scale, layer0=0):
    """q [n_layers, B, Hq, d]; codes / z / s for the whole cache as
    codec.encode_block_uniform lays them out ([L, 2, B, H, T/16, d/16, ...]);
    G [L, 2, H, d/16, 16, 16].  Returns [n_layers, B, Hq, d] (fp64)."""
    nl = q.shape[0]
    nb = n_tokens // 16
    sl = slice(layer0, layer0 + nl)
    x = _codec.decode_block_uniform(codes[sl, :, :, :, :nb], z[sl, :, :, :, :nb], s[sl, :, :, :, :nb],
                                    np.asarray(G, np.float64)[sl], bits)   # [nl, 2, B, H, n, d]
    return softmax_attention(q, x[:, 0], x[:, 1], scale)
