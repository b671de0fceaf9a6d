"""GPU parity of the grouped-gauge block-uniform codec against the oracle.

Codes, scales and zero points must match the oracle's quantizer bit for bit,
given the gauged values the kernel quantized: the fp32 FMA chain (g = 8, 32,
16 x d ranges, the CUDA-core engine), which must itself match the oracle's
chain bit for bit, or the default g = 16 engine's own two-term tensor-core
contraction, which must lie within 2^-16 sum_j |G_ij x_j| of the exact G x.
Decoded reconstructions must match the oracle's fp64 G^T (s q + z) within the
bf16 tolerance (per-slice norm-relative 2e-3 plus an elementwise half-ulp bound).
"""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import gauge as og
from oracle import quant as oq
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import (assert_close_bf16, assert_gauge_within, bf16_np, block_uniform_np, chain_tensor_g16,
                            need_gpu, oracle_quantize_own, own_gauge_g16, run_decode, run_encode)

pytestmark = pytest.mark.gpu


def oracle_gauge(A):
    """fp32 G = exp(A - A^T) from the oracle (both sides then read the same G)."""
    return torch.from_numpy(og.gauge_from_A(A.cpu().numpy().astype(np.float64)).astype(np.float32)).cuda()


def _inputs(L, B, H, T, d, g, seed=0, sigma=0.1, n_outliers=None, outliers=(3, 17)):
    kv = synth.kv_cache(L, B, H, T, d, seed=seed, device="cuda", outlier_channels=outliers, n_outliers=n_outliers)
    A = synth.gauge_params(L, H, d // g, g, sigma=sigma, seed=seed)
    return kv, A, oracle_gauge(A)


def _check_encode(kv, G, codec, t0=0, nt=None):
    """Encode on the GPU and check it against the oracle.  Chain engines: codes,
    steps, zero points and gauged values equal the oracle's fp32 chain.  The
    default g = 16 engine: codes, steps and zero points equal the oracle's
    quantizer applied to the kernel's own gauged values, which lie within the
    two-term tensor-core bound of the exact G x.  Returns the reference codes
    (equal to the device's) for the decode check."""
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    x = bf16_np(kv)
    G32 = G.cpu().numpy().astype(np.float64)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    y = gauged.cpu().numpy().astype(np.float64)
    if own_gauge_g16(kv.shape, codec):
        assert_gauge_within(y[..., t0:t0 + nt, :], x[..., t0:t0 + nt, :], G32, what="gauged values")
        ref = oracle_quantize_own(y[..., t0:t0 + nt, :], codec.bits, codec.range_cols)
    else:
        ref = oc.encode_block_uniform(x, G32, codec.bits, tb=16, w=codec.range_cols, t0=t0, nt=nt)
        if chain_tensor_g16(kv.shape, codec):
            # the chain-exact tensor-core encoder reports the values it quantized: within
            # 2^-16 of the block maximum from the chain (its codes are the chain's)
            d = oq.block_uniform_view(np.abs(y[..., t0:t0 + nt, :] - ref["y"]), 16, 16).max(-1)
            m = oq.block_uniform_view(np.abs(ref["y"]), 16, 16).max(-1)
            assert np.all(d <= 2.0 ** -16 * m), "gauged values beyond the tensor-core bound"
        else:
            assert np.array_equal(y[..., t0:t0 + nt, :], ref["y"]), "gauged values differ from the fp32 chain"
    assert np.all(np.isnan(y[..., :t0, :])) and np.all(np.isnan(y[..., t0 + nt:, :])), "wrote outside the range"
    assert np.array_equal(z[..., tb0:tb1, :], np.asarray(ref["z"]).astype(np.float16).view(np.uint16))
    assert np.array_equal(s[..., tb0:tb1, :], np.asarray(ref["s"]).astype(np.float16).view(np.uint16))
    assert np.array_equal(c[..., tb0:tb1, :, :], ref["codes"])
    assert not c[..., :tb0, :, :].any() and not c[..., tb1:, :, :].any(), "codes written outside the range"
    return codes, scales, zeros, ref


@pytest.mark.parametrize("bits", [3, 4, 6])
def test_tiny_config_encode_decode(bits):
    """The small reference cache: 1 layer, 2 KV heads, d=64, 1024 tokens, g=16."""
    need_gpu()
    kv, A, G = _inputs(1, 1, 2, 1024, 64, 16)
    codec = cg.codec_desc(g=16, bits=bits)
    codes, scales, zeros, ref = _check_encode(kv, G, codec)
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G.cpu().numpy().astype(np.float64), bits)
    assert_close_bf16(bf16_np(out), xr, what="decode")


@pytest.mark.parametrize("g,bits,wfull", [(8, 2, False), (8, 3, True), (16, 8, False), (16, 4, True), (16, 3, True),
                                          (32, 4, False), (32, 6, True), (8, 6, False), (32, 2, False)])
def test_group_sizes_bits_and_range_widths(g, bits, wfull):
    need_gpu()
    d = 128
    kv, A, G = _inputs(2, 2, 2, 96, d, g, seed=g + bits)
    codec = cg.codec_desc(g=g, bits=bits, range_cols=d if wfull else g)
    codes, scales, zeros, ref = _check_encode(kv, G, codec)
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G.cpu().numpy().astype(np.float64), bits,
                                 w=codec.range_cols)
    assert_close_bf16(bf16_np(out), xr, what="decode g=%d b=%d" % (g, bits))


@pytest.mark.parametrize("t0,nt", [(0, 16), (48, 32), (80, 176), (240, 16)])
def test_token_ranges_append(t0, nt):
    """Rolling append: only blocks of [t0, t0+nt) are written (ragged tails of a pass)."""
    need_gpu()
    kv, A, G = _inputs(1, 1, 3, 256, 64, 16, seed=5)
    codec = cg.codec_desc(g=16, bits=4)
    codes, scales, zeros, ref = _check_encode(kv, G, codec, t0, nt)
    out = run_decode(kv.shape, G, codec, codes, scales, zeros, t0, nt, fill=7.0)
    o = bf16_np(out)
    assert np.all(o[..., :t0, :] == 7.0) and np.all(o[..., t0 + nt:, :] == 7.0)
    xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G.cpu().numpy().astype(np.float64), 4)
    assert_close_bf16(o[..., t0:t0 + nt, :], xr, what="decode range")


def test_identity_gauge_is_plain_quantizer_and_degenerate_blocks():
    need_gpu()
    kv = synth.kv_cache(1, 1, 2, 64, 64, seed=3, device="cuda")
    kv[0, 0, 0, 0, :16, :] = 1.5            # constant block: s = 0, q = 0
    kv[0, 1, 0, 1, 16:32, :16] = 0.0        # zero block
    kv[0, 1, 0, 0, 32:48, :] *= 1000.0      # large values
    G = synth.identity_gauge(1, 2, 4, 16, device="cuda")
    codec = cg.codec_desc(g=16, bits=4)
    codes, scales, zeros, ref = _check_encode(kv, G, codec)
    q, z, s = oq.quantize_ranges(oq.block_uniform_view(bf16_np(kv), 16, 16), 4)
    assert np.array_equal(ref["q"], q)
    c, sb, zb = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    assert sb[0, 0, 0, 0, 0, 0] == 0 and not c[0, 0, 0, 0, 0, 0].any()
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    assert np.all(bf16_np(out)[0, 0, 0, 0, :16, :16] == 1.5)


def test_gauge_build_group_and_full_head():
    """cg_gauge_build against the oracle's fp64 exp(A - A^T), fp64 internals rounded once
    to fp32 (at g = 128 the scaled skew matrix is held in fp32): max-abs error and
    orthogonality |G^T G - I| within 1e-5 at every g (1e-6 / 4e-6 for g <= 64), including
    a g = 128 set whose norm needs several squarings, g = 96 (padded to 128) and g = 12 and
    36 (padded to the next multiple of 8 for the fp64 tensor-core products)."""
    need_gpu()
    for g, sigma, n, tol, otol in [(8, 0.1, 64, 1e-6, 4e-6), (16, 0.1, 512, 1e-6, 4e-6), (32, 0.1, 64, 1e-6, 4e-6),
                                   (12, 0.1, 32, 1e-6, 4e-6), (36, 0.05, 8, 1e-6, 4e-6),
                                   (64, 0.05, 16, 1e-6, 4e-6), (128, 0.05, 16, 1e-5, 1e-5), (128, 0.5, 4, 1e-5, 1e-5),
                                   (96, 0.05, 4, 1e-5, 1e-5)]:
        A = torch.randn(n, g, g, generator=torch.Generator().manual_seed(g)) * sigma
        G = torch.empty_like(A).cuda()
        cg.cg_gauge_build(A.cuda(), G)
        Gd = G.cpu().numpy().astype(np.float64)
        Gref = og.gauge_from_A(A.numpy().astype(np.float64))
        assert np.abs(Gd - Gref).max() < tol, (g, sigma, np.abs(Gd - Gref).max())
        eye = np.einsum("nji,njk->nik", Gd, Gd)
        assert np.abs(eye - np.eye(g)).max() < otol, (g, sigma, np.abs(eye - np.eye(g)).max())


@pytest.mark.slow
@pytest.mark.parametrize("bits", [3, 4, 6])
def test_8b_shaped_cache_sampled_parity(bits):
    """Full 8B-shaped cache (32 x 2 x 8 x 4096 x 128) in the launch configuration the
    benchmark times (no gauged output): its codes equal those of a second run that
    also writes the gauged values, and on sampled (l, s, h) slices the oracle checks
    them (its quantizer on those gauged values), the gauged values themselves and the
    decode."""
    need_gpu()
    L, B, H, T, d = 32, 1, 8, 4096, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=1, device="cuda", n_outliers=4)
    G = oracle_gauge(synth.gauge_params(L, H, d // 16, 16, sigma=0.1, seed=1))
    codec = cg.codec_desc(g=16, bits=bits)
    codes, scales, zeros, _ = run_encode(kv, G, codec, want_gauged=False)
    codes2, scales2, zeros2, gauged = run_encode(kv, G, codec, want_gauged=True)
    assert torch.equal(codes, codes2) and torch.equal(scales, scales2) and torch.equal(zeros, zeros2)
    del codes2, scales2, zeros2
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    rng = np.random.default_rng(bits)
    for _ in range(3):
        l, sk, h = int(rng.integers(L)), int(rng.integers(2)), int(rng.integers(H))
        x = bf16_np(kv[l:l + 1, sk:sk + 1, :, h:h + 1])
        Gs = G[l:l + 1, sk:sk + 1, h:h + 1].cpu().numpy().astype(np.float64)
        y = gauged[l:l + 1, sk:sk + 1, :, h:h + 1].cpu().numpy().astype(np.float64)
        assert_gauge_within(y, x, Gs, what="8B slice gauged values")
        ref = oracle_quantize_own(y, bits, 16)
        assert np.array_equal(c[l, sk, :, h], ref["codes"][0, 0, :, 0])
        assert np.array_equal(s[l, sk, :, h], ref["s"][0, 0, :, 0].astype(np.float16).view(np.uint16))
        assert np.array_equal(z[l, sk, :, h], ref["z"][0, 0, :, 0].astype(np.float16).view(np.uint16))
        xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], Gs, bits)
        assert_close_bf16(bf16_np(out[l:l + 1, sk:sk + 1, :, h:h + 1]), xr, what="8B slice")
