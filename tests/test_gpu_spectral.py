"""GPU parity of the spectral training statistics against the oracle (fp64):
per-block L_freq and L_rate within 1e-4 relative (floor 1e-3 for L_freq ~ 0),
totals within 1e-4 relative, dL/dG within 1e-4 Frobenius-relative."""
import numpy as np
import pytest
import torch

from oracle import spectral as sp
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import bf16_np, need_gpu
from tests.test_gpu_codec import oracle_gauge

pytestmark = pytest.mark.gpu


def run_stats(x, G, want_grad, x_is_fp32):
    L, _, B, H, T, d = x.shape
    kvd = cg.kv_desc(L, B, H, T, d)
    st = cg.StatsDesc(16, 16 if G is not None else 0, int(x_is_fp32), 1.0, 0.02, 0.04)
    nblk = L * 2 * B * H * T // 16
    lf = torch.empty(nblk, dtype=torch.float32, device="cuda")
    lr = torch.empty_like(lf)
    tot = torch.empty(4, dtype=torch.float64, device="cuda")
    dG = torch.empty_like(G) if want_grad else None
    ws_bytes = cg.cg_spectral_workspace_size(kvd, st, want_grad)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    cg.cg_spectral_stats(kvd, st, x, G, lf, lr, tot, dG, ws)
    cg.cg_sync_status()
    return lf.cpu().numpy(), lr.cpu().numpy(), tot.cpu().numpy(), None if dG is None else dG.cpu().numpy()


def _check(ref, lf, lr, tot, dG=None):
    rl, rr = ref["lfreq"].reshape(-1), ref["lrate"].reshape(-1)
    assert np.all(np.abs(lf - rl) <= 1e-4 * np.maximum(np.abs(rl), 1e-3)), np.abs(lf - rl).max()
    assert np.all(np.abs(lr - rr) <= 1e-4 * np.maximum(np.abs(rr), 1e-3)), np.abs(lr - rr).max()
    rt = ref["totals"]
    assert tot[2] == rt[2]
    assert np.all(np.abs(tot - rt) <= 1e-4 * np.abs(rt)), (tot, rt)
    if dG is not None:
        rel = np.sqrt(((dG - ref["dG"]) ** 2).sum() / (ref["dG"] ** 2).sum())
        assert rel <= 1e-4, rel


@pytest.mark.parametrize("want_grad", [False, True])
def test_stats_bf16_cache_with_gauge(want_grad):
    need_gpu()
    L, B, H, T, d = 2, 2, 2, 256, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=4, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=4))
    lf, lr, tot, dG = run_stats(kv, G, want_grad, False)
    ref = sp.spectral_stats(bf16_np(kv), G.cpu().numpy().astype(np.float64), want_grad=want_grad)
    _check(ref, lf, lr, tot, dG)


def test_stats_fp32_gauged_input():
    """x already gauged (fp32), no G: the stats pass of the training windows."""
    need_gpu()
    L, B, H, T, d = 1, 1, 3, 384, 128
    g = torch.Generator().manual_seed(5)
    x = (torch.randn((L, 2, B, H, T, d), generator=g) * 3).cuda()
    x[0, 0, 0, 1, 16:32] = 0.0          # an all-zero block: L_freq = L_rate = 0
    x[0, 1, 0, 2, 32:48] = 1.25         # a constant block: L_freq = 0
    lf, lr, tot, _ = run_stats(x, None, False, True)
    ref = sp.spectral_stats(x.cpu().numpy().astype(np.float64), None)
    _check(ref, lf, lr, tot)
    nb = T // 16
    assert lf[(0 * 2 + 0) * H * nb + 1 * nb + 1] == 0.0 and lr[(0 * 2 + 0) * H * nb + 1 * nb + 1] == 0.0
    assert abs(lf[(0 * 2 + 1) * H * nb + 2 * nb + 2]) < 1e-6


def test_stats_identity_gauge_matches_ungauged():
    need_gpu()
    kv = synth.kv_cache(1, 1, 2, 128, 128, seed=7, device="cuda")
    I = synth.identity_gauge(1, 2, 8, 16, device="cuda")
    lf1, lr1, t1, dG = run_stats(kv, I, True, False)
    lf0, lr0, t0, _ = run_stats(kv.float().contiguous(), None, False, True)
    assert np.allclose(lf1, lf0, rtol=1e-5, atol=1e-7) and np.allclose(lr1, lr0, rtol=1e-5, atol=1e-7)
    ref = sp.spectral_stats(bf16_np(kv), np.broadcast_to(np.eye(16), (1, 2, 2, 8, 16, 16)).copy(), want_grad=True)
    _check(ref, lf1, lr1, t1, dG)


@pytest.mark.slow
def test_stats_window_8b_sampled():
    """One 4096-token window of the 8B-shaped cache (fp32 gauged input, 1.07 GB) with the
    gradient through a g = 16 gauge on the bf16 cache: totals and sampled blocks."""
    need_gpu()
    L, B, H, T, d = 32, 1, 8, 4096, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=3, device="cuda", n_outliers=4)
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=3))
    lf, lr, tot, dG = run_stats(kv, G, True, False)
    # oracle on a few (l, s, h) slices: per-block values, and dG of those gauge sets
    rng = np.random.default_rng(1)
    nb = T // 16
    for _ in range(2):
        l, s, h = int(rng.integers(L)), int(rng.integers(2)), int(rng.integers(H))
        x = bf16_np(kv[l:l + 1, s:s + 1, :, h:h + 1])
        Gs = G[l:l + 1, s:s + 1, h:h + 1].cpu().numpy().astype(np.float64)
        ref = sp.spectral_stats(x, Gs)
        base = ((l * 2 + s) * B * H + h) * nb
        rl, rr = ref["lfreq"].reshape(-1), ref["lrate"].reshape(-1)
        assert np.all(np.abs(lf[base:base + nb] - rl) <= 1e-4 * np.maximum(np.abs(rl), 1e-3))
        assert np.all(np.abs(lr[base:base + nb] - rr) <= 1e-4 * np.maximum(np.abs(rr), 1e-3))
    assert tot[2] == L * 2 * B * H * nb
    lam_r = float(np.float32(0.02))  # lambda_r crosses the C ABI as fp32
    assert abs(tot[3] - (tot[0] / tot[2] + lam_r * tot[1] / tot[2])) <= 1e-12 * abs(tot[3])
    assert np.isfinite(dG).all() and np.abs(dG).max() > 0
