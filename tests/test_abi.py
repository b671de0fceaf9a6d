"""The C-ABI library loads, exports every entry point include/cg.h declares, and
its host-side validation rejects bad arguments before any CUDA call (these
tests pass fake, never-dereferenced pointers and run without a GPU)."""
import ctypes
import os
import re

import pytest

from quantization_cg_encode_b200 import cg

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "cg.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cg_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert "cg_encode" in names and "cg_decode" in names and "cg_spectral_stats" in names
    L = cg.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(cg.EXPORTS)


def test_version_and_status_strings():
    assert cg.cg_version() >= 100
    assert cg.status_string(cg.CG_OK) == "ok"
    assert "invalid" in cg.status_string(cg.CG_ERR_INVALID)
    assert "timed out" in cg.status_string(cg.CG_ERR_TIMEOUT)
    assert "error bound" in cg.status_string(cg.CG_ERR_BOUND)


@pytest.mark.parametrize("bits,g,w", [(3, 16, 16), (4, 16, 16), (6, 16, 16), (4, 16, 128), (4, 128, 128), (2, 8, 8)])
def test_sizes_closed_form(bits, g, w):
    kvd = cg.kv_desc(32, 1, 8, 4096, 128)
    cb, sc = cg.cg_sizes_for(kvd, cg.codec_desc(g=g, bits=bits, range_cols=w))
    n = 32 * 2 * 8 * 4096 * 128
    assert cb == n * bits // 8
    assert sc == 32 * 2 * 8 * (4096 // 16) * (128 // w)
    assert 8 * (cb + 4 * sc) / n == pytest.approx(bits + 32 / (16 * w))


def test_sizes_kivi():
    kvd = cg.kv_desc(2, 1, 2, 256, 128)
    cb, sc = cg.cg_sizes_for(kvd, cg.codec_desc(g=16, bits=3, mode=cg.KIVI))
    n = 2 * 2 * 2 * 256 * 128
    assert cb == n * 3 // 8 and sc == n // 32


def _enc(kvd, codec, kv=0x10000, G=0x20000, t0=0, nt=0, codes=0x30000, sc=0x40000, z=0x50000, gauged=None):
    L = cg.lib()
    vp = ctypes.c_void_p
    return L.cg_encode(ctypes.byref(kvd), ctypes.byref(codec), vp(kv), vp(G), t0, nt, vp(codes), vp(sc), vp(z),
                       None if gauged is None else vp(gauged), None)


def test_encode_validation_without_gpu():
    kvd = cg.kv_desc(1, 1, 2, 1024, 64)
    ok = cg.codec_desc(g=16, bits=4)
    assert _enc(kvd, ok, nt=0) == cg.CG_OK                                 # empty range: no launch
    assert _enc(kvd, ok, nt=16, kv=0) == cg.CG_ERR_INVALID                 # null input
    assert _enc(kvd, ok, nt=16, codes=0x30008) == cg.CG_ERR_INVALID        # misaligned
    assert _enc(kvd, ok, nt=16, gauged=0x60004) == cg.CG_ERR_INVALID       # misaligned optional
    assert _enc(kvd, ok, t0=8, nt=16) == cg.CG_ERR_INVALID                 # off the 16-token grid
    assert _enc(kvd, ok, t0=1024, nt=16) == cg.CG_ERR_INVALID              # beyond capacity
    assert _enc(kvd, ok, nt=-16) == cg.CG_ERR_INVALID
    assert _enc(kvd, cg.codec_desc(g=16, bits=5), nt=16) == cg.CG_ERR_UNSUPPORTED
    assert _enc(kvd, cg.codec_desc(g=24, bits=4), nt=16) == cg.CG_ERR_INVALID
    assert _enc(kvd, cg.codec_desc(g=16, bits=4, range_cols=24), nt=16) == cg.CG_ERR_INVALID
    assert _enc(kvd, cg.codec_desc(g=16, bits=4, tb=8), nt=16) == cg.CG_ERR_UNSUPPORTED
    assert _enc(cg.kv_desc(1, 1, 2, 1000, 64), ok, nt=0) == cg.CG_ERR_INVALID  # T not a multiple of 32
    assert _enc(cg.kv_desc(1, 1, 2, 1024, 96), cg.codec_desc(g=16, bits=4), nt=0) == cg.CG_ERR_UNSUPPORTED
    kivi = cg.codec_desc(g=16, bits=3, mode=cg.KIVI)
    assert _enc(kvd, kivi, t0=16, nt=32) == cg.CG_ERR_INVALID              # KIVI needs 32-token steps
    assert _enc(kvd, cg.codec_desc(g=16, bits=4, engine=7), nt=16) == cg.CG_ERR_INVALID   # unknown engine
    chain_tc = cg.codec_desc(g=16, bits=4, engine=cg.ENGINE_CHAIN_TENSOR)
    assert _enc(cg.kv_desc(1, 1, 2, 1024, 64), chain_tc, nt=16) == cg.CG_ERR_UNSUPPORTED  # d = 128 only
    chain_w = cg.codec_desc(g=16, bits=4, range_cols=128, engine=cg.ENGINE_CHAIN_TENSOR)
    assert _enc(cg.kv_desc(1, 1, 2, 1024, 128), chain_w, nt=16) == cg.CG_ERR_UNSUPPORTED  # 16 x 16 ranges only
    full = cg.codec_desc(g=128, bits=4, range_cols=128, engine=cg.ENGINE_CUDA_CORES)
    assert _enc(cg.kv_desc(1, 1, 2, 1024, 128), full, nt=16) == cg.CG_ERR_UNSUPPORTED  # full head: tensor cores only


def test_decode_and_build_validation_without_gpu():
    L = cg.lib()
    vp = ctypes.c_void_p
    kvd = cg.kv_desc(1, 1, 2, 1024, 64)
    c = cg.codec_desc(g=16, bits=4)
    r = L.cg_decode(ctypes.byref(kvd), ctypes.byref(c), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), 0, 0,
                    vp(0x5000), None)
    assert r == cg.CG_OK
    r = L.cg_decode(ctypes.byref(kvd), ctypes.byref(c), vp(0x1000), vp(0x2000), vp(0x3000), vp(0), 0, 16,
                    vp(0x5000), None)
    assert r == cg.CG_ERR_INVALID
    assert L.cg_gauge_build(vp(0x1000), vp(0x1000), 4, 16, None) == cg.CG_ERR_INVALID   # aliasing
    assert L.cg_gauge_build(vp(0x1000), vp(0x2000), 4, 200, None) == cg.CG_ERR_INVALID  # g too large
    assert L.cg_gauge_build(vp(0x1000), vp(0x2000), 0, 16, None) == cg.CG_OK            # nothing to do


def test_selftest_validation_without_gpu():
    L = cg.lib()
    vp = ctypes.c_void_p
    assert L.cg_selftest_wait_timeout(0, vp(0x1000), None) == cg.CG_ERR_INVALID           # no limit
    assert L.cg_selftest_wait_timeout(3000000000, vp(0x1000), None) == cg.CG_ERR_INVALID  # above 2 s
    assert L.cg_selftest_wait_timeout(1000000, vp(0), None) == cg.CG_ERR_INVALID          # null result


def test_attention_validation_without_gpu():
    L = cg.lib()
    kvd = cg.kv_desc(2, 1, 2, 512, 128)
    bad = [cg.AttnDesc(5, 512, 0, 1, 0.1),    # Hq not a multiple of H
           cg.AttnDesc(6 * 2, 512, 0, 1, 0.1),  # group of 6
           cg.AttnDesc(4, 500, 0, 1, 0.1),    # n not a multiple of 16
           cg.AttnDesc(4, 528, 0, 1, 0.1),    # n beyond T
           cg.AttnDesc(4, 512, 1, 2, 0.1),    # layers beyond L
           cg.AttnDesc(4, 512, 0, 1, 0.0)]    # scale
    out = ctypes.c_uint64()
    codes = [cg.CG_ERR_INVALID, cg.CG_ERR_UNSUPPORTED, cg.CG_ERR_INVALID, cg.CG_ERR_INVALID, cg.CG_ERR_INVALID,
             cg.CG_ERR_INVALID]
    for at, want in zip(bad, codes):
        assert L.cg_decode_attention_workspace_size(ctypes.byref(kvd), ctypes.byref(at), ctypes.byref(out)) == want


def _rt(kvd, codec, kv=0x10000, G=0x20000, codes=0x30000, sc=0x40000, z=0x50000, out=0x60000, ws=0x70000,
        ws_bytes=1 << 40):
    L = cg.lib()
    vp = ctypes.c_void_p
    return L.cg_roundtrip_host(ctypes.byref(kvd), ctypes.byref(codec), vp(kv), vp(G), vp(codes), vp(sc), vp(z),
                               vp(out), vp(ws), ws_bytes, None)


def test_roundtrip_workspace_and_validation_without_gpu():
    kvd = cg.kv_desc(32, 1, 8, 4096, 128)
    assert cg.cg_roundtrip_workspace_size(kvd) == 4 * 2 * 8 * 4096 * 128 * 2   # four one-layer bf16 buffers
    ok = cg.codec_desc(g=16, bits=4)
    assert _rt(kvd, ok, kv=0) == cg.CG_ERR_INVALID                        # null host input
    assert _rt(kvd, ok, out=0) == cg.CG_ERR_INVALID                       # null host output
    assert _rt(kvd, ok, codes=0x30008) == cg.CG_ERR_INVALID               # misaligned device output
    assert _rt(kvd, ok, ws=0x70004) == cg.CG_ERR_INVALID                  # misaligned workspace
    assert _rt(kvd, ok, ws_bytes=cg.cg_roundtrip_workspace_size(kvd) - 16) == cg.CG_ERR_INVALID
    assert _rt(kvd, cg.codec_desc(g=16, bits=5)) == cg.CG_ERR_UNSUPPORTED
    # one layer's steps with 16 x d ranges: 2 B H (T / 16) fp16 = 8 bytes here, not a multiple of 16
    assert _rt(cg.kv_desc(2, 1, 1, 32, 64), cg.codec_desc(g=16, bits=4, range_cols=64)) == cg.CG_ERR_UNSUPPORTED
