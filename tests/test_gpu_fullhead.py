"""Full-head gauge (g = d_head = 128) on the tensor cores: y = G_bf16 x per token
with fp32 accumulation.  The gauged values must match the oracle's exact
G_bf16 x within the fp32 accumulation bound; codes, scales and zero points must
equal, bit for bit, the oracle's quantizer applied to the kernel's own fp32
gauged output (the quantizer given the same fp32 gauged input), and the
oracle's decisions on the exact values wherever those are unique under the
bound; reconstructions within the bf16 tolerance.

Launch geometry: both kernels are persistent, one CTA per SM (148 on a B200),
over 128-token blocks of every head slice.  The encoder streams blocks through a
4-stage ring into four TMEM accumulators that three epilogue warpgroups take in
turn; the decoder's two warpgroups take alternate blocks and load the next
block's codes early.  The many-blocks cases give each CTA 7 to 28 blocks, so the
ring wraps, every accumulator and warpgroup is reused, G is restaged across head
slices and the decoder's early loads run."""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import gauge as og
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import (assert_close_bf16, bf16_np, block_uniform_np, check_block_codes_valid, need_gpu,
                            oracle_quantize_own, run_decode, run_encode)

pytestmark = pytest.mark.gpu


def _gauge(kind, L, H, seed):
    if kind == "expm":
        A = synth.gauge_params(L, H, 1, 128, sigma=0.05, seed=seed)
        return torch.from_numpy(og.gauge_from_A(A.numpy().astype(np.float64)).astype(np.float32)).cuda()
    if kind == "identity":
        return synth.identity_gauge(L, H, 1, 128, device="cuda")
    if kind == "haar":
        return synth.haar_gauge(L, H, 1, 128, seed=seed, device="cuda")
    return synth.dct_gauge(L, H, 1, 128, device="cuda")


def _encode_check(kv, G, bits, t0=0, nt=None):
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    codec = cg.codec_desc(g=128, bits=bits, range_cols=128)
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    x = bf16_np(kv)[..., t0:t0 + nt, :]
    Gb = og.round_gauge_bf16(G.cpu().numpy().astype(np.float64))
    y_ref = og.apply_gauge(x, Gb)
    # |fp32 accumulation of 128 exact products - exact sum| <= 128 u sum|G x| (u = 2^-24), doubled for margin
    eps = 2 * 128 * 2.0 ** -24 * og.apply_gauge(np.abs(x), np.abs(Gb)) + 1e-30
    y = gauged.cpu().numpy().astype(np.float64)[..., t0:t0 + nt, :]
    assert np.all(np.abs(y - y_ref) <= eps), "gauged values beyond the fp32 accumulation bound"
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    # bit-exact: the oracle's quantizer on the kernel's own gauged values
    own = oracle_quantize_own(y, bits, 128)
    assert np.array_equal(c[..., tb0:tb1, :, :], own["codes"]), "codes differ from the oracle quantizer of y"
    assert np.array_equal(s[..., tb0:tb1, :], np.asarray(own["s"]).astype(np.float16).view(np.uint16)), "steps"
    assert np.array_equal(z[..., tb0:tb1, :], np.asarray(own["z"]).astype(np.float16).view(np.uint16)), "zeros"
    assert not c[..., :tb0, :, :].any() and not c[..., tb1:, :, :].any(), "codes written outside the range"
    # and the oracle's own decisions on the exact values wherever they are unique
    n, amb = check_block_codes_valid(c[..., tb0:tb1, :, :], s[..., tb0:tb1, :], z[..., tb0:tb1, :], y_ref, eps, bits, 128)
    assert amb <= max(32, n // 100), "too many undecidable codes: %d of %d" % (amb, n)
    return codec, codes, scales, zeros, Gb


@pytest.mark.parametrize("kind,bits", [("expm", 4), ("identity", 4), ("haar", 3), ("dct", 6)])
def test_fullhead_encode(kind, bits):
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 512, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=3, device="cuda")
    G = _gauge(kind, L, H, seed=bits)
    _encode_check(kv, G, bits)


def test_fullhead_identity_is_plain_quantizer_exactly():
    """With G = I every product but one is zero, so the tensor-core sum is exact:
    codes must equal the plain quantizer's bit for bit."""
    need_gpu()
    kv = synth.kv_cache(1, 1, 2, 256, 128, seed=8, device="cuda")
    G = _gauge("identity", 1, 2, 0)
    codec = cg.codec_desc(g=128, bits=4, range_cols=128)
    codes, scales, zeros, gauged = run_encode(kv, G, codec)
    ref = oc.encode_block_uniform(bf16_np(kv), G.cpu().numpy().astype(np.float64), 4, w=128, full_head_bf16=True)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    assert np.array_equal(gauged.cpu().numpy(), bf16_np(kv))
    assert np.array_equal(c, ref["codes"])
    assert np.array_equal(s, np.asarray(ref["s"]).astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("t0,nt", [(128, 256), (48, 80), (0, 16)])
def test_fullhead_token_ranges(t0, nt):
    need_gpu()
    kv = synth.kv_cache(1, 2, 2, 384, 128, seed=5, device="cuda")
    G = _gauge("expm", 1, 2, seed=5)
    _encode_check(kv, G, 4, t0, nt)


@pytest.mark.parametrize("kind,bits,t0,nt", [("expm", 4, 0, None), ("haar", 3, 0, None), ("dct", 6, 128, 256),
                                             ("identity", 8, 48, 80), ("expm", 2, 0, None)])
def test_fullhead_decode(kind, bits, t0, nt):
    """x_hat = G_bf16^T (s q + z) on the tensor cores vs the oracle's fp64 value, both
    decoding the codes, steps and zero points the oracle's own encoder produced."""
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 512, 128
    nt = T - t0 if nt is None else nt
    kv = synth.kv_cache(L, B, H, T, d, seed=6, device="cuda")
    G = _gauge(kind, L, H, seed=bits)
    ref = oc.encode_block_uniform(bf16_np(kv), G.cpu().numpy().astype(np.float64), bits, w=128, t0=t0, nt=nt,
                                  full_head_bf16=True)
    codec = cg.codec_desc(g=128, bits=bits, range_cols=128)
    kvd = cg.kv_desc_of(kv)
    codes, scales, zeros = cg.alloc_encoded(kvd, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    cv = codes.view(L, 2, B, H, T // 16, 1, 16 * d * bits // 8)
    cv[:, :, :, :, tb0:tb1] = torch.from_numpy(ref["codes"]).cuda()
    scales.view(L, 2, B, H, T // 16, 1)[:, :, :, :, tb0:tb1] = torch.from_numpy(ref["s"].astype(np.float16)).cuda()
    zeros.view(L, 2, B, H, T // 16, 1)[:, :, :, :, tb0:tb1] = torch.from_numpy(ref["z"].astype(np.float16)).cuda()
    out = run_decode(kv.shape, G, codec, codes, scales, zeros, t0, nt, fill=3.0)
    xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G.cpu().numpy().astype(np.float64), bits, w=128,
                                 full_head_bf16=True)
    o = bf16_np(out)
    assert np.all(o[..., :t0, :] == 3.0) and np.all(o[..., t0 + nt:, :] == 3.0)
    assert_close_bf16(o[..., t0:t0 + nt, :], xr, what="full-head decode")


def _decode_own_check(kv, G, Gb, codec, codes, scales, zeros, bits, t0, nt, slices):
    """Decode the kernel's own (verified) codes; compare sampled slices with the
    oracle's fp64 G_bf16^T (s q + z)."""
    L, _, B, H, T, d = kv.shape
    out = run_decode(kv.shape, G, codec, codes, scales, zeros, t0, nt, fill=3.0)
    o = bf16_np(out)
    assert np.all(o[..., :t0, :] == 3.0) and np.all(o[..., t0 + nt:, :] == 3.0), "decode wrote outside the range"
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    from oracle import gauge as _og
    from oracle import quant as _oq
    for l, sk, h in slices:
        q = _oq.unpack_codes(c[l, sk, :, h, tb0:tb1], bits, 16 * 128)
        zz = s[l, sk, :, h, tb0:tb1].view(np.float16).astype(np.float64)  # steps
        z0 = z[l, sk, :, h, tb0:tb1].view(np.float16).astype(np.float64)
        yhat = _oq.block_uniform_unview(_oq.dequantize(q, z0[..., None], zz[..., None]), 16, 128)
        xr = _og.apply_inverse_gauge(yhat[None, None, :, None], Gb[l:l + 1, sk:sk + 1, h:h + 1])
        assert_close_bf16(o[l:l + 1, sk:sk + 1, :, h:h + 1, t0:t0 + nt], xr, what="full-head decode %s" % ((l, sk, h),))


@pytest.mark.parametrize("kind,bits", [("expm", 4), ("identity", 3), ("haar", 6), ("dct", 4)])
def test_fullhead_many_blocks_per_cta(kind, bits):
    """4 x 2 x 4 x 4096 x 128 with t0 = 32 and a ragged end (nt = 4096 - 80): 1024
    blocks of 128 tokens, about 7 per CTA, crossing head slices; every gauge kind."""
    need_gpu()
    L, B, H, T, d = 4, 1, 4, 4096, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=21, device="cuda", n_outliers=4)
    G = _gauge(kind, L, H, seed=bits)
    t0, nt = 32, T - 80
    codec, codes, scales, zeros, Gb = _encode_check(kv, G, bits, t0, nt)
    _decode_own_check(kv, G, Gb, codec, codes, scales, zeros, bits, t0, nt, [(0, 0, 0), (3, 1, 3), (1, 1, 2)])


def test_fullhead_deep_schedule():
    """8 x 2 x 8 x 4096 x 128 (the benchmark's per-layer shape, 8 layers): 4096 blocks,
    about 28 per CTA, so the 4-stage ring wraps 7 times and each of the four TMEM
    accumulators is reused 7 times; every code checked, decode on sampled slices."""
    need_gpu()
    L, B, H, T, d = 8, 1, 8, 4096, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=23, device="cuda", n_outliers=4)
    G = _gauge("expm", L, H, seed=23)
    codec, codes, scales, zeros, Gb = _encode_check(kv, G, 4, 0, T)
    _decode_own_check(kv, G, Gb, codec, codes, scales, zeros, 4, 0, T, [(0, 0, 0), (7, 1, 7), (4, 0, 5)])
