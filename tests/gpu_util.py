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
