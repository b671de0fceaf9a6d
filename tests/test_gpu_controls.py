"""Coordinate controls on the GPU: the per-group Gram matrices (cg_group_gram,
fp64) against the oracle, the KLT gauge built from them, and the Hadamard and
KLT gauges through the codec (codes bit-exact against the oracle quantizer of
the kernel's gauged values; decode within the bf16 tolerance)."""
import numpy as np
import pytest
import torch

from oracle import codec as ocd
from oracle import controls as oc
from quantization_cg_encode_b200 import cg, controls, synth
from tests.gpu_util import (assert_close_bf16, assert_gauge_within, bf16_np, block_uniform_np, need_gpu,
                            oracle_quantize_own, run_decode, run_encode)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,g,t0,nt", [(128, 16, 0, None), (128, 8, 32, 200), (128, 32, 0, 64), (64, 16, 16, 96)])
def test_group_gram_matches_oracle(d, g, t0, nt):
    need_gpu()
    L, B, H, T = 2, 3, 2, 256
    kv = synth.kv_cache(L, B, H, T, d, seed=g + d, device="cuda", n_outliers=2)
    kvd = cg.kv_desc_of(kv)
    gram = torch.full((L, 2, H, d // g, g, g), float("nan"), dtype=torch.float64, device="cuda")
    cg.cg_group_gram(kvd, g, kv, gram, t0, nt)
    cg.cg_sync_status()
    ref = oc.gram(bf16_np(kv), g, t0, nt)
    got = gram.cpu().numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("kind", ["hadamard", "klt"])
def test_control_gauges_through_the_codec(kind):
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 512, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=7, device="cuda", n_outliers=2)
    if kind == "hadamard":
        G = controls.hadamard_gauge(L, H, d // 16, 16, device="cuda")
        assert np.allclose(G[0, 0, 0, 0].cpu().numpy(), oc.hadamard(16), atol=1e-7)
    else:
        G = controls.klt_gauge(kv, 16)
        ref_G, w = oc.klt(oc.gram(bf16_np(kv), 16))
        Gn = G.cpu().numpy().astype(np.float64)
        assert np.allclose(Gn, ref_G, atol=1e-5)          # the same basis, up to fp32 rounding
        C = oc.gram(bf16_np(kv), 16)
        D = np.einsum("lshrij,lshrjk,lshrmk->lshrim", Gn, C, Gn)
        off = D - np.einsum("...ii->...i", D)[..., None] * np.eye(16)
        assert np.abs(off).max() <= 1e-5 * np.abs(D).max()  # second moments decorrelated
    codec = cg.codec_desc(g=16, bits=4)
    codes, scales, zeros, gauged = run_encode(kv, G, codec)
    y = gauged.cpu().numpy().astype(np.float64)
    G64 = G.cpu().numpy().astype(np.float64)
    assert_gauge_within(y, bf16_np(kv), G64, what=kind)
    ref = oracle_quantize_own(y, 4, 16)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    assert np.array_equal(c, ref["codes"])
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    xr = ocd.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G64, 4)
    assert_close_bf16(bf16_np(out), xr, what=kind + " decode")
