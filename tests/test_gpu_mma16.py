"""GPU parity of the default g = 16 codec (16 x 16 block-uniform ranges,
d_head 64 and 128): the warp-level tensor-core encoder and decoder.

The encoder's gauged values are its own tensor-core contraction with G split
into two bf16 terms.  Codes, steps and zero points must equal, bit for bit, the
oracle's quantizer applied to those fp32 gauged values (the quantizer given the
same fp32 gauged input); the gauged values must lie within 2^-16 sum_j |G_ij x_j|
of the oracle's exact G x.  The decoder must match the oracle's fp64
G^T (s q + z) of the same codes within the bf16 tolerance.

Launch geometry: both kernels are persistent, one CTA per SM (148 on a B200),
16 warps.  The encoder streams 256-token stages through a ring of 3 (d = 128)
or 6 (d = 64); the decoder 256-token (d = 128) or 512-token (d = 64) stages
through a ring of 8 (5 when a stage's codes exceed 24 KB).  The many-stage cases
below give every CTA several times its ring depth in stages, crossing head
slices (G fragments reloaded) and ragged slice ends.
"""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import gauge as og
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import (assert_close_bf16, assert_gauge_within, bf16_np, block_uniform_np, need_gpu,
                            oracle_quantize_own, run_decode, run_encode)

pytestmark = pytest.mark.gpu


def _gauge(L, H, d, seed, sigma=0.1):
    A = synth.gauge_params(L, H, d // 16, 16, sigma=sigma, seed=seed)
    return og.gauge_from_A(A.numpy().astype(np.float64)).astype(np.float32)


def _roundtrip(kv, G32, bits, t0=0, nt=None, decode_slices=None):
    """Encode + decode through the C ABI; check everything against the oracle."""
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    G = torch.from_numpy(G32).cuda()
    codec = cg.codec_desc(g=16, bits=bits)
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    x = bf16_np(kv)
    y = gauged.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(y[..., :t0, :])) and np.all(np.isnan(y[..., t0 + nt:, :])), "gauged written outside"
    y = y[..., t0:t0 + nt, :]
    assert_gauge_within(y, x[..., t0:t0 + nt, :], G32.astype(np.float64), what="gauged values")
    ref = oracle_quantize_own(y, bits, 16)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    assert np.array_equal(z[..., tb0:tb1, :], np.asarray(ref["z"]).astype(np.float16).view(np.uint16)), "zero points"
    assert np.array_equal(s[..., tb0:tb1, :], np.asarray(ref["s"]).astype(np.float16).view(np.uint16)), "steps"
    assert np.array_equal(c[..., tb0:tb1, :, :], ref["codes"]), "codes"
    assert not c[..., :tb0, :, :].any() and not c[..., tb1:, :, :].any(), "codes written outside the range"
    out = run_decode(kv.shape, G, codec, codes, scales, zeros, t0, nt, fill=7.0)
    o = bf16_np(out)
    assert np.all(o[..., :t0, :] == 7.0) and np.all(o[..., t0 + nt:, :] == 7.0), "decode wrote outside the range"
    o = o[..., t0:t0 + nt, :]
    G64 = G32.astype(np.float64)
    if decode_slices is None:
        xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G64, bits)
        assert_close_bf16(o, xr, what="decode")
    else:
        for l, sk, h in decode_slices:
            xr = oc.decode_block_uniform(ref["codes"][l:l + 1, sk:sk + 1, :, h:h + 1],
                                         ref["z"][l:l + 1, sk:sk + 1, :, h:h + 1],
                                         ref["s"][l:l + 1, sk:sk + 1, :, h:h + 1],
                                         G64[l:l + 1, sk:sk + 1, h:h + 1], bits)
            assert_close_bf16(o[l:l + 1, sk:sk + 1, :, h:h + 1], xr, what="decode slice %s" % ((l, sk, h),))
    return codes, scales, zeros


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_bits_and_head_widths(bits, d):
    need_gpu()
    kv = synth.kv_cache(2, 2, 2, 512, d, seed=bits + d, device="cuda", n_outliers=4)
    _roundtrip(kv, _gauge(2, 2, d, seed=bits), bits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("t0,nt", [(0, 16), (48, 176), (16, 240), (128, 128), (0, 400), (272, 144)])
def test_ragged_token_ranges(d, t0, nt):
    """Partial stages at the end of every head slice; only [t0, t0 + nt) is written."""
    need_gpu()
    kv = synth.kv_cache(1, 1, 3, 416, d, seed=7, device="cuda", n_outliers=2)
    _roundtrip(kv, _gauge(1, 3, d, seed=7), 4, t0, nt)


@pytest.mark.parametrize("bits", [3, 4])
def test_many_stages_per_cta(bits):
    """8 x 2 x 8 x 4096 x 128 with a ragged end per slice (nt = 4096 - 48): 2048
    encoder stages (about 14 per CTA, the 3-deep ring wraps 4 times) and 2048 decoder
    stages (about 14 per CTA, the 8-deep ring wraps), every CTA crossing head slices.
    Codes checked everywhere; decode on sampled slices."""
    need_gpu()
    L, H, T, d = 8, 8, 4096, 128
    kv = synth.kv_cache(L, 1, H, T, d, seed=11 + bits, device="cuda", n_outliers=4)
    rng = np.random.default_rng(bits)
    sl = [(int(rng.integers(L)), int(rng.integers(2)), int(rng.integers(H))) for _ in range(4)]
    _roundtrip(kv, _gauge(L, H, d, seed=11), bits, 0, T - 48, decode_slices=sl)


def test_many_stages_d64():
    """d = 64: 12 x 2 x 8 x 4096 with t0 = 32 and a ragged end per slice: about 21
    encoder stages per CTA (ring of 6) and 10 decoder stages (ring of 8)."""
    need_gpu()
    L, H, T, d = 12, 8, 4096, 64
    kv = synth.kv_cache(L, 1, H, T, d, seed=5, device="cuda", n_outliers=4)
    _roundtrip(kv, _gauge(L, H, d, seed=5), 4, 32, T - 96, decode_slices=[(0, 0, 0), (11, 1, 7), (5, 1, 2)])


def test_degenerate_blocks_and_clamping():
    """Identity gauge (the gauged values are the inputs, exactly): constant and zero
    blocks (step 0); a block below -65504 (the zero point clamps to -65504, so low
    codes clamp to 0); a block spanning +-1e6 (the step saturates at 65504, so codes
    clamp at both ends); values in the fp16 subnormal range (zero point rounded
    relative to a tiny range); values on rounding ties; large magnitudes; a block of
    -0 (stored as +0 step and zero point); then a non-orthogonal gauge."""
    need_gpu()
    L, B, H, T, d = 1, 1, 2, 256, 128
    rng = np.random.default_rng(3)
    x = rng.standard_normal((L, 2, B, H, T, d)).astype(np.float32)
    x[0, 0, 0, 0, :16, :] = 1.5                                   # constant block
    x[0, 0, 0, 0, 16:32, :] = 0.0                                 # zero block
    x[0, 0, 0, 0, 32:48, :] = -1e5 - 512.0 * rng.integers(0, 4, (16, d))   # below the fp16 range
    x[0, 0, 0, 0, 48:64, :] = 1e6 * np.sign(rng.standard_normal((16, d)))  # step saturates
    x[0, 0, 0, 0, 64:80, :] = 3e-7 * rng.standard_normal((16, d))          # fp16 subnormal range
    k = rng.integers(0, 30, size=(16, d)).astype(np.float32)
    x[0, 0, 0, 1, :16, :] = -1.0 + 0.125 * k                      # ties at odd k (4-bit grid)
    x[0, 0, 0, 1, 0, :] = -1.0
    x[0, 0, 0, 1, 1, :] = 2.75
    x[0, 1, 0, 0] *= 3000.0                                       # large magnitudes
    x[0, 1, 0, 1, :16, :16] = -0.0                                # a block of -0
    kv = torch.from_numpy(x).to(torch.bfloat16).cuda()
    eye = np.broadcast_to(np.eye(16, dtype=np.float32), (L, 2, H, 8, 16, 16)).copy()
    for bits in (3, 4, 8):
        codes, scales, zeros = _roundtrip(kv, eye, bits)
        c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, cg.codec_desc(g=16, bits=bits))
        assert s[0, 0, 0, 0, 0, 0] == 0 and not c[0, 0, 0, 0, 0, 0].any()  # constant block: step 0, codes 0
        assert s[0, 0, 0, 0, 1, 0] == 0 and z[0, 0, 0, 0, 1, 0] == 0         # zero block: +0 step and zero point
        assert s[0, 1, 0, 1, 0, 0] == 0 and z[0, 1, 0, 1, 0, 0] == 0         # -0 block: +0 as well
        assert z[0, 0, 0, 0, 2, 0] == np.float16(-65504).view(np.uint16)    # clamped zero point
        if bits < 8:                                                         # 2e6 / (2^b - 1) > 65504
            assert s[0, 0, 0, 0, 3, 0] == np.float16(65504).view(np.uint16)  # saturated step
    G32 = _gauge(L, H, d, seed=13)
    G32[0, 0] *= 1.5
    G32[0, 1] = rng.standard_normal(G32[0, 1].shape).astype(np.float32) * 0.3
    _roundtrip(kv, G32, 4)


def test_gauged_output_does_not_change_codes():
    """The benchmark launches without the gauged output: the codes must be those of
    the launch that reports it."""
    need_gpu()
    kv = synth.kv_cache(4, 1, 8, 1024, 128, seed=17, device="cuda", n_outliers=4)
    G = torch.from_numpy(_gauge(4, 8, 128, seed=17)).cuda()
    codec = cg.codec_desc(g=16, bits=4)
    a = run_encode(kv, G, codec, want_gauged=False)
    b = run_encode(kv, G, codec, want_gauged=True)
    for u, v in zip(a[:3], b[:3]):
        assert torch.equal(u, v)
