"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
bring its outputs to numpy for comparison with the oracle."""
import numpy as np
import pytest
import torch

from quantization_cg_encode_b200 import cg


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cg.lib()  # a missing library is an error, not a skip


def bf16_np(t):
    """bf16 torch tensor -> float64 numpy (exact)."""
    return t.float().cpu().numpy().astype(np.float64)


def fp16_bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def run_encode(kv, G, codec, t0=0, nt=None, want_gauged=True):
    kvd = cg.kv_desc_of(kv)
    nt = kvd.tokens - t0 if nt is None else nt
    codes, scales, zeros = cg.alloc_encoded(kvd, codec, device=kv.device)
    gauged = torch.full(kv.shape, float("nan"), dtype=torch.float32, device=kv.device) if want_gauged else None
    cg.cg_encode(kvd, codec, kv, G, t0, nt, codes, scales, zeros, gauged)
    cg.cg_sync_status()
    return codes, scales, zeros, gauged


def run_decode(kv_shape, G, codec, codes, scales, zeros, t0=0, nt=None, fill=0.0):
    kvd = cg.KvDesc(kv_shape[0], kv_shape[2], kv_shape[3], kv_shape[4], kv_shape[5])
    nt = kvd.tokens - t0 if nt is None else nt
    out = torch.full(kv_shape, fill, dtype=torch.bfloat16, device=codes.device)
    cg.cg_decode(kvd, codec, codes, scales, zeros, G, t0, nt, out)
    cg.cg_sync_status()
    return out


def chain_tensor_g16(shape, codec):
    """True when cg_encode runs the chain-exact tensor-core g = 16 encoder."""
    return codec.engine == cg.ENGINE_CHAIN_TENSOR


def own_gauge_g16(shape, codec):
    """True when cg_encode's gauged values are its own two-term tensor-core
    contraction (the default engine for g = 16 with 16 x 16 ranges)."""
    return (codec.g == 16 and shape[-1] in (64, 128) and codec.range_cols == 16 and codec.mode == cg.BLOCK_UNIFORM
            and codec.engine == cg.ENGINE_AUTO)


def oracle_quantize_own(y, bits, w):
    """The oracle's block-uniform quantizer applied to the device's fp32 gauged
    values y [..., T, d]: dict(codes, z, s, q) in the oracle's layout."""
    from oracle import quant as oq
    q, z, s = oq.quantize_ranges(oq.block_uniform_view(np.asarray(y, np.float64), 16, w), bits)
    return dict(codes=oq.pack_codes(q, bits), z=z, s=s, q=q)


def kivi_own_gauge(shape, codec):
    """True when cg_encode's KIVI-style gauged values are its own two-term
    tensor-core contraction (the default engine for g = 16, d_head 64 or 128)."""
    return codec.mode == cg.KIVI and codec.g == 16 and shape[-1] in (64, 128) and codec.engine == cg.ENGINE_AUTO


def oracle_kivi_own(y, bits):
    """The oracle's KIVI-style quantizer (keys per channel over 32 tokens, values per
    token over 32 channels) applied to the device's fp32 gauged values y
    [L, 2, B, H, nt, d]: the layout of oracle.codec.encode_kivi's result."""
    from oracle import quant as oq
    y = np.asarray(y, np.float64)
    qk, zk, sk = oq.quantize_ranges(oq.kivi_key_view(y[:, 0], 32), bits)
    qv, zv, sv = oq.quantize_ranges(oq.kivi_value_view(y[:, 1], 32), bits)
    return dict(key=dict(codes=oq.pack_codes(qk, bits), z=zk, s=sk, q=qk),
                value=dict(codes=oq.pack_codes(qv, bits), z=zv, s=sv, q=qv), y=y)


OWN_GAUGE_BOUND = 2.0 ** -16


def assert_gauge_within(y_dev, x, G, bound=OWN_GAUGE_BOUND, what=""):
    """|y_dev - G x| <= bound * sum_j |G_ij x_j| for every value (G x exact, fp64),
    and the per-slice norm-relative error far inside 2e-3."""
    from oracle import gauge as og
    y_dev = np.asarray(y_dev, np.float64)
    ref = og.apply_gauge(x, G)
    mag = og.apply_gauge(np.abs(x), np.abs(np.asarray(G, np.float64)))
    err = np.abs(y_dev - ref)
    bad = err > bound * mag
    assert not bad.any(), "%s: %d gauged values beyond %.3g sum|G x|, worst ratio %.3g" % (
        what, int(bad.sum()), bound, float((err / np.maximum(mag, 1e-300)).max()))
    flat_e = (y_dev - ref).reshape(-1, ref.shape[-2] * ref.shape[-1])
    flat_r = ref.reshape(flat_e.shape)
    rel = np.sqrt((flat_e ** 2).sum(-1)) / np.maximum(np.sqrt((flat_r ** 2).sum(-1)), 1e-300)
    assert rel.max() <= 2e-3, "%s: slice norm-relative error %.3g" % (what, rel.max())


def block_uniform_np(codes, scales, zeros, shape, codec):
    """Device buffers -> numpy views [L,2,B,H,T/16,d/W,bytes] and [L,2,B,H,T/16,d/W]."""
    L, _, B, H, T, d = shape
    W = codec.range_cols
    nb = 16 * W * codec.bits // 8
    c = codes.cpu().numpy().reshape(L, 2, B, H, T // 16, d // W, nb)
    s = fp16_bits(scales).reshape(L, 2, B, H, T // 16, d // W)
    z = fp16_bits(zeros).reshape(L, 2, B, H, T // 16, d // W)
    return c, s, z


def assert_close_bf16(got, ref, rel_norm=2e-3, what=""):
    """Reconstruction tolerance: per (l,s,b,h) slice ||got-ref|| / ||ref|| <= rel_norm,
    and elementwise |got-ref| <= 2^-8 |ref| (half a bf16 ulp) + 1e-4 rms(ref)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    flat_g = got.reshape(-1, got.shape[-2] * got.shape[-1])
    flat_r = ref.reshape(flat_g.shape)
    num = np.sqrt(((flat_g - flat_r) ** 2).sum(-1))
    den = np.sqrt((flat_r ** 2).sum(-1))
    worst = (num / np.maximum(den, 1e-300)).max()
    assert worst <= rel_norm, "%s: slice norm-relative error %.3g > %.3g" % (what, worst, rel_norm)
    rms = np.sqrt((flat_r ** 2).mean(-1, keepdims=True))
    bound = 2.0 ** -8 * np.abs(flat_r) + 1e-4 * rms
    bad = np.abs(flat_g - flat_r) > bound
    assert not bad.any(), "%s: %d elements beyond the bf16 bound, worst %.3g" % (
        what, int(bad.sum()), float((np.abs(flat_g - flat_r) - bound).max()))


def kivi_np(codes, scales, zeros, shape, bits):
    """Device KIVI buffers -> (keys, values) numpy views matching the oracle's layout."""
    L, _, B, H, T, d = shape
    per = T * d * bits // 8
    c = codes.cpu().numpy().reshape(L, 2, B, H, per)
    nr = T * d // 32
    s = fp16_bits(scales).reshape(L, 2, B, H, nr)
    z = fp16_bits(zeros).reshape(L, 2, B, H, nr)
    keys = dict(codes=c[:, 0].reshape(L, B, H, T // 32, d, 4 * bits), s=s[:, 0].reshape(L, B, H, T // 32, d),
                z=z[:, 0].reshape(L, B, H, T // 32, d))
    vals = dict(codes=c[:, 1].reshape(L, B, H, T, d // 32, 4 * bits), s=s[:, 1].reshape(L, B, H, T, d // 32),
                z=z[:, 1].reshape(L, B, H, T, d // 32))
    return keys, vals


def check_block_codes_valid(c, s_bits, z_bits, y_ref, eps, bits, w):
    """Codes from a tensor-core gauge: y is only defined to +-eps (fp32 accumulation
    order is the hardware's), so each decision must be the oracle's exact one
    wherever the oracle's value is more than eps from a rounding boundary, and a
    valid rounding of some y' in [y - eps, y + eps] everywhere else.

    c      : [..., nblk, bytes] packed codes, s_bits / z_bits : [..., nblk] fp16 bits
    y_ref  : [..., T, d] exact gauged values (fp64), eps : [..., T, d] bound
    Returns (n_values, n_values whose decision was not unique).
    """
    from oracle import quant as oq
    from oracle.fpround import fl16, fl32, F16_MAX
    qmax = 2 ** bits - 1
    yb = oq.block_uniform_view(np.asarray(y_ref, np.float64), 16, w)
    eb = oq.block_uniform_view(np.asarray(eps, np.float64), 16, w)
    q = oq.unpack_codes(c, bits, 16 * w)
    zg = np.asarray(z_bits, np.uint16).view(np.float16).astype(np.float64)
    sg = np.asarray(s_bits, np.uint16).view(np.float16).astype(np.float64)
    em = eb.max(axis=-1)
    mn, mx = yb.min(axis=-1), yb.max(axis=-1)
    zlo = fl16(np.clip(fl32(mn - em), -F16_MAX, F16_MAX))
    zhi = fl16(np.clip(fl32(mn + em), -F16_MAX, F16_MAX))
    assert np.all((zg >= zlo) & (zg <= zhi)), "zero point outside its admissible interval"
    slo = fl16(np.minimum(fl32(fl32(np.maximum(mx - mn - 2 * em, 0)) / qmax), F16_MAX))
    shi = fl16(np.minimum(fl32(fl32(mx - mn + 2 * em) / qmax), F16_MAX))
    assert np.all((sg >= slo) & (sg <= shi)), "step outside its admissible interval"
    q_lo = oq.quantize(fl32(yb - eb), zg[..., None], sg[..., None], bits)
    q_hi = oq.quantize(fl32(yb + eb), zg[..., None], sg[..., None], bits)
    assert np.all((q >= q_lo) & (q <= q_hi)), "code outside its admissible interval"
    # given the device's (validated) z and s, a code is decided uniquely when its interval is one value
    unique = q_lo == q_hi
    q_ref = oq.quantize(fl32(yb), zg[..., None], sg[..., None], bits)
    assert np.array_equal(q[unique], q_ref[unique])
    # z and s themselves must be the oracle's wherever their intervals are single values
    z_ref, s_ref = oq.quant_params(mn, mx, bits)
    assert np.array_equal(zg[zlo == zhi], z_ref[zlo == zhi]) and np.array_equal(sg[slo == shi], s_ref[slo == shi])
    return q.size, int((~unique).sum())
