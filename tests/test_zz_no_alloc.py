"""The allocation-free spectral-statistics entry point.

Some callers of this library cannot allocate device memory (serving engines
with a fixed memory plan, plug-ins given only pre-planned buffers, real-time
loops that must avoid cudaMalloc's implicit synchronization).  For them
cg_spectral_stats_noalloc takes no workspace and keeps its dL/dG partials in a
scratch array built into the library.  These tests call it through the C ABI
twice in a row and compare every output with cg_spectral_stats (caller
workspace), within the tolerances the spectral tests use, and check that
requests larger than the built-in scratch are refused.  This file is collected
last on purpose, so that a failing run stopped at the first failure has
already run every other test; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantization_cg_encode_b200 import cg, synth

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cg.lib()


def _outputs(kvd, like_G, nblk):
    lf = torch.full((nblk,), float("nan"), dtype=torch.float32, device="cuda")
    lr = torch.full_like(lf, float("nan"))
    tot = torch.full((4,), float("nan"), dtype=torch.float64, device="cuda")
    dG = torch.full_like(like_G, float("nan"))
    return lf, lr, tot, dG


def _close(a, b, rel=1e-4, floor=1e-3):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.all(np.abs(a - b) <= rel * np.maximum(np.abs(b), floor))


def test_noalloc_matches_workspace_entry_point_twice():
    _need_gpu()
    L, B, H, T, d = 2, 2, 2, 256, 128           # 16 head slices, within the built-in limit
    kv = synth.kv_cache(L, B, H, T, d, seed=21, device="cuda")
    A = synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=21).cuda()
    G = torch.empty_like(A)
    cg.cg_gauge_build(A, G)
    kvd = cg.kv_desc(L, B, H, T, d)
    st = cg.StatsDesc(16, 16, 0, 1.0, 0.02, 0.04)
    nblk = L * 2 * B * H * T // 16
    ref = _outputs(kvd, G, nblk)
    ws = torch.empty(cg.cg_spectral_workspace_size(kvd, st, True), dtype=torch.uint8, device="cuda")
    cg.cg_spectral_stats(kvd, st, kv, G, *ref, ws)
    for _ in range(2):                          # two calls in a row share the scratch array
        got = _outputs(kvd, G, nblk)
        cg.cg_spectral_stats_noalloc(kvd, st, kv, G, *got)
        cg.cg_sync_status()
        for g_, r_ in zip(got, ref):
            assert torch.isfinite(g_).all()
        assert _close(got[0], ref[0]) and _close(got[1], ref[1])
        assert _close(got[2], ref[2], rel=1e-4, floor=0.0)
        rel = torch.linalg.norm((got[3] - ref[3]).double()) / torch.linalg.norm(ref[3].double())
        assert rel <= 1e-4


def test_noalloc_forward_only_and_limit():
    _need_gpu()
    L, B, H, T, d = 1, 1, 2, 128, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=22, device="cuda")
    kvd = cg.kv_desc(L, B, H, T, d)
    st = cg.StatsDesc(16, 0, 0, 1.0, 0.02, 0.04)
    x = kv.float().contiguous()
    st32 = cg.StatsDesc(16, 0, 1, 1.0, 0.02, 0.04)
    nblk = L * 2 * B * H * T // 16
    lf = torch.empty(nblk, dtype=torch.float32, device="cuda")
    lr, tot = torch.empty_like(lf), torch.empty(4, dtype=torch.float64, device="cuda")
    lf2, lr2, tot2 = torch.empty_like(lf), torch.empty_like(lf), torch.empty_like(tot)
    cg.cg_spectral_stats(kvd, st32, x, None, lf, lr, tot, None, None)
    cg.cg_spectral_stats_noalloc(kvd, st32, x, None, lf2, lr2, tot2)
    cg.cg_sync_status()
    assert _close(lf2, lf) and _close(lr2, lr) and _close(tot2, tot, floor=0.0)
    # a request needing more scratch than is built in is refused before any launch:
    # 40 x 2 x 1 x 8 = 640 head slices of 256 tokens (two dG partials of 8 KB each) > 8 MiB
    big = cg.kv_desc(40, 1, 8, 256, 128)
    stg = cg.StatsDesc(16, 16, 0, 1.0, 0.02, 0.04)
    vp = ctypes.c_void_p
    r = cg.lib().cg_spectral_stats_noalloc(ctypes.byref(big), ctypes.byref(stg), vp(0x10000), vp(0x20000),
                                           vp(0x30000), vp(0x40000), vp(0x50000), vp(0x60000), None)
    assert r == cg.CG_ERR_TOO_LARGE
    assert "scratch" in cg.status_string(r)
