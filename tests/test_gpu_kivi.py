"""GPU parity of the KIVI-style codec (keys per channel over 32 tokens, values
per token over 32 channels) with the grouped gauge fused, against the oracle:
codes, scales and zero points bit-exact against the oracle's quantizer given the
gauged values (for the fp32 chain engine, the oracle's own chain; for the
default g = 16 engine, the kernel's tensor-core gauged values, which are checked
against G x within 2^-16 sum |G x|); reconstructions within the bf16 tolerance;
rolling append of 128-token chunks identical to a one-shot encode."""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import (assert_close_bf16, assert_gauge_within, bf16_np, kivi_np, kivi_own_gauge, need_gpu,
                            oracle_kivi_own, run_decode, run_encode)
from tests.test_gpu_codec import oracle_gauge

pytestmark = pytest.mark.gpu


def _f16bits(a):
    return np.asarray(a).astype(np.float16).view(np.uint16)


def _check(kv, G, bits, g, t0=0, nt=None, engine=cg.ENGINE_AUTO):
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    codec = cg.codec_desc(g=g, bits=bits, mode=cg.KIVI, engine=engine)
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    G32 = G.cpu().numpy().astype(np.float64)
    y = gauged.cpu().numpy().astype(np.float64)[..., t0:t0 + nt, :]
    if kivi_own_gauge(kv.shape, codec):
        assert_gauge_within(y, bf16_np(kv)[..., t0:t0 + nt, :], G32, what="kivi gauged values")
        ref = oracle_kivi_own(y, bits)
    else:
        ref = oc.encode_kivi(bf16_np(kv), G32, bits, t0=t0, nt=nt)
        assert np.array_equal(y, ref["y"])
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


@pytest.mark.parametrize("g,bits,engine", [(16, 3, cg.ENGINE_AUTO), (16, 4, cg.ENGINE_AUTO), (8, 2, cg.ENGINE_AUTO),
                                           (32, 6, cg.ENGINE_AUTO), (16, 8, cg.ENGINE_AUTO), (8, 3, cg.ENGINE_AUTO),
                                           (16, 3, cg.ENGINE_CUDA_CORES), (16, 4, cg.ENGINE_CUDA_CORES),
                                           (16, 2, cg.ENGINE_AUTO), (16, 6, cg.ENGINE_AUTO)])
def test_kivi_parity(g, bits, engine):
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 128, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=g * 10 + bits, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, d // g, g, sigma=0.1, seed=bits))
    _check(kv, G, bits, g, engine=engine)


@pytest.mark.parametrize("d,bits,T,t0,nt", [(128, 3, 2048, 0, 2048), (128, 4, 1024, 96, 800), (64, 3, 2048, 32, 1984)])
def test_kivi_default_engine_many_units(d, bits, T, t0, nt):
    """The default g = 16 engine over several units per CTA: 8 x 2 x 4 slices of up to 2048
    tokens in units of 8192 / d tokens (2048 units at d = 128 over at most 3 CTAs per SM;
    a ragged last unit; a start inside the first unit) against the oracle quantizer of its
    own gauged values."""
    need_gpu()
    L, B, H = 8, 1, 4
    kv = synth.kv_cache(L, B, H, T, d, seed=d + bits + t0, device="cuda", n_outliers=2)
    G = oracle_gauge(synth.gauge_params(L, H, d // 16, 16, sigma=0.1, seed=bits))
    _check(kv, G, bits, 16, t0=t0, nt=nt)


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
    g = 16 fused, default engine (no gauged output at this size): full encode + decode.
    On sampled (layer, head, 4096-token window) slices: the same window encoded on its
    own with the gauged output gives the same bytes (the kernel's values depend only on
    the slice and its gauge), and that encode matches the oracle quantizer of its own
    gauged values; the decode matches the oracle decode of those codes."""
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
        win = kv[l:l + 1, :, :, h:h + 1, t0:t0 + 4096].contiguous()
        Gw = G[l:l + 1, :, h:h + 1].contiguous()
        c1, s1, z1, y1 = run_encode(win, Gw, codec)
        k1, v1 = kivi_np(c1, s1, z1, win.shape, bits)
        assert np.array_equal(keys["codes"][l, :, h, t0 // 32:(t0 + 4096) // 32], k1["codes"][0, :, 0])
        assert np.array_equal(vals["codes"][l, :, h, t0:t0 + 4096], v1["codes"][0, :, 0])
        assert np.array_equal(keys["s"][l, :, h, t0 // 32:(t0 + 4096) // 32], k1["s"][0, :, 0])
        assert np.array_equal(vals["z"][l, :, h, t0:t0 + 4096], v1["z"][0, :, 0])
        Gs = Gw.cpu().numpy().astype(np.float64)
        y = y1.cpu().numpy().astype(np.float64)
        assert_gauge_within(y, bf16_np(win), Gs, what="long-context window")
        ref = oracle_kivi_own(y, bits)
        assert np.array_equal(k1["codes"], ref["key"]["codes"])
        assert np.array_equal(v1["codes"], ref["value"]["codes"])
        assert np.array_equal(k1["s"], _f16bits(ref["key"]["s"]))
        assert np.array_equal(v1["z"], _f16bits(ref["value"]["z"]))
        xr = oc.decode_kivi(ref, Gs, bits)
        assert_close_bf16(bf16_np(out[l:l + 1, :, :, h:h + 1, t0:t0 + 4096]), xr, what="long-context slice")
