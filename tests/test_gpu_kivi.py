"""GPU parity of the KIVI-style codec (keys per channel over 32 tokens, values
per token over 32 channels) with the grouped gauge fused, against the oracle:
codes, scales and zero points bit-exact; reconstructions within the bf16
tolerance; rolling append of 128-token chunks identical to a one-shot encode."""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import assert_close_bf16, bf16_np, kivi_np, need_gpu, run_decode, run_encode
from tests.test_gpu_codec import oracle_gauge

pytestmark = pytest.mark.gpu


def _f16bits(a):
    return np.asarray(a).astype(np.float16).view(np.uint16)


def _check(kv, G, bits, g, t0=0, nt=None):
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    codec = cg.codec_desc(g=g, bits=bits, mode=cg.KIVI)
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    G32 = G.cpu().numpy().astype(np.float64)
    ref = oc.encode_kivi(bf16_np(kv), G32, bits, t0=t0, nt=nt)
    y = gauged.cpu().numpy().astype(np.float64)
    assert np.array_equal(y[..., t0:t0 + nt, :], ref["y"])
    keys, vals = kivi_np(codes, scales, zeros, kv.shape, bits)
    g0, g1 = t0 // 32, (t0 + nt) // 32
    assert np.array_equal(keys["codes"][:, :, :, g0:g1], ref["key"]["codes"])
    assert np.array_equal(keys["s"][:, :, :, g0:g1], _f16bits(ref["key"]["s"]))
    assert np.array_equal(keys["z"][:, :, :, g0:g1], _f16bits(ref["key"]["z"]))
    assert np.array_equal(vals["codes"][:, :, :, t0:t0 + nt], ref["value"]["codes"])
    assert np.array_equal(vals["s"][:, :, :, t0:t0 + nt], _f16bits(ref["value"]["s"]))
    assert np.array_equal(vals["z"][:, :, :, t0:t0 + nt], _f16bits(ref["value"]["z"]))
    out = run_decode(kv.shape, G, codec, codes, scales, zeros, t0, nt)
    xr = oc.decode_kivi(ref, G32, bits)
    assert_close_bf16(bf16_np(out)[..., t0:t0 + nt, :], xr, what="kivi decode")
    return codes, scales, zeros


@pytest.mark.parametrize("g,bits", [(16, 3), (16, 4), (8, 2), (32, 6), (16, 8), (8, 3)])
def test_kivi_parity(g, bits):
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 128, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=g * 10 + bits, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, d // g, g, sigma=0.1, seed=bits))
    _check(kv, G, bits, g)


def test_kivi_tiny_d64_ranges():
    need_gpu()
    kv = synth.kv_cache(1, 1, 2, 256, 64, seed=4, device="cuda")
    G = oracle_gauge(synth.gauge_params(1, 2, 4, 16, sigma=0.1, seed=4))
    _check(kv, G, 3, 16, t0=64, nt=96)


def test_kivi_rolling_append_matches_one_shot():
    """128-token chunks appended one by one give the bytes of a one-shot encode."""
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 640, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=9, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=9))
    codec = cg.codec_desc(g=16, bits=3, mode=cg.KIVI)
    kvd = cg.kv_desc_of(kv)
    one = cg.alloc_encoded(kvd, codec)
    cg.cg_encode(kvd, codec, kv, G, 0, T, *one)
    roll = cg.alloc_encoded(kvd, codec)
    cg.cg_encode(kvd, codec, kv, G, 0, 128, *roll)          # prefill
    for t0 in range(128, T, 128):                               # decode steps append chunks
        cg.cg_encode(kvd, codec, kv, G, t0, 128, *roll)
    cg.cg_sync_status()
    for a, b in zip(one, roll):
        assert torch.equal(a, b)
    _check(kv, G, 3, 16, t0=256, nt=128)


@pytest.mark.slow
def test_long_context_kivi_sampled_parity():
    """The long-context cache (48 x 2 x 8 x 131072 x 128 bf16, 25.8 GB) at 3 bits with
    g = 16 fused: full encode + decode, oracle on sampled (layer, K/V, head) slices."""
    need_gpu()
    L, B, H, T, d, bits = 48, 1, 8, 131072, 128, 3
    free, _ = torch.cuda.mem_get_info()
    if free < 70e9:
        pytest.skip("needs ~60 GB of device memory")
    kv = synth.kv_cache(L, B, H, T, d, seed=2, device="cuda", n_outliers=4)
    G = oracle_gauge(synth.gauge_params(L, H, d // 16, 16, sigma=0.1, seed=2))
    codec = cg.codec_desc(g=16, bits=bits, mode=cg.KIVI)
    codes, scales, zeros, _ = run_encode(kv, G, codec, want_gauged=False)
    out = run_decode(kv.shape, G, codec, codes, scales, zeros)
    keys, vals = kivi_np(codes, scales, zeros, kv.shape, bits)
    rng = np.random.default_rng(0)
    for _ in range(2):
        l, h = int(rng.integers(L)), int(rng.integers(H))
        t0 = int(rng.integers(0, T // 4096)) * 4096
        x = bf16_np(kv[l:l + 1, :, :, h:h + 1, t0:t0 + 4096])
        Gs = G[l:l + 1, :, h:h + 1].cpu().numpy().astype(np.float64)
        ref = oc.encode_kivi(x, Gs, bits)
        assert np.array_equal(keys["codes"][l, :, h, t0 // 32:(t0 + 4096) // 32], ref["key"]["codes"][0, :, 0])
        assert np.array_equal(vals["codes"][l, :, h, t0:t0 + 4096], ref["value"]["codes"][0, :, 0])
        assert np.array_equal(keys["s"][l, :, h, t0 // 32:(t0 + 4096) // 32], _f16bits(ref["key"]["s"][0, :, 0]))
        assert np.array_equal(vals["z"][l, :, h, t0:t0 + 4096], _f16bits(ref["value"]["z"][0, :, 0]))
        xr = oc.decode_kivi(ref, Gs, bits)
        assert_close_bf16(bf16_np(out[l:l + 1, :, :, h:h + 1, t0:t0 + 4096]), xr, what="long-context slice")
