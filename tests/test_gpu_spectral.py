"""GPU parity of the spectral training statistics against the oracle (fp64):
per-block L_freq and L_rate within 1e-4 relative (floor 1e-3 for L_freq ~ 0),
totals within 1e-4 relative, dL/dG within 1e-4 Frobenius-relative (where the
rate proxy's kink at U = 0 can matter, plus the bound of what sign decisions at
the kink can change; see rate_kink_allowance).  d_head = 128
with whole 128-token tiles runs the tensor-core kernel; d_head = 64 and other
token counts run the CUDA-core kernel."""
import numpy as np
import pytest
import torch

from oracle import spectral as sp
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import bf16_np, need_gpu
from tests.test_gpu_codec import oracle_gauge

pytestmark = pytest.mark.gpu


def run_stats(x, G, want_grad, x_is_fp32, lambda_f=1.0, lambda_r=0.02):
    L, _, B, H, T, d = x.shape
    kvd = cg.kv_desc(L, B, H, T, d)
    st = cg.StatsDesc(16, 16 if G is not None else 0, int(x_is_fp32), lambda_f, lambda_r, 0.04)
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


def rate_kink_allowance(x, G, n_blocks_total, lambda_r=0.02, tau=0.04, rel_eps=2.0 ** -16):
    """Frobenius allowance, per gauge set [L, 2, H], for the dL/dG difference that
    sign decisions at the rate proxy's kink can make.

    d log(1 + |U|/tau) / dU = sign(U) / (tau + |U|) jumps by 2 / tau at U = 0 (the
    oracle takes sign(0) = 0).  A coefficient within the device's rounding of zero
    may land on either side, changing dU_uv by up to c = 2 lambda_r / (tau N_U).
    "Within rounding of zero" is |U| <= rel_eps * rms(U of the block): the device
    carries X' and dU_1 as bf16 hi + lo pairs (2^-17 relative), so its U differs from
    the exact one by about 2^-17 of the block's norm, i.e. 2^-17 sqrt(16 d) of the
    block's rms coefficient.

    One such coefficient (u, v) of block k changes dG_r[i][j] by
    c C_d[v][16 r + i] W_k[u][16 r + j] with W_k = C_16 x_k (the token DCT of x), so
    its exact Frobenius size is c (sum_r |C_d[v, group r]|^2 |W_k[u, group r]|^2)^(1/2).
    The sides the coefficients take are independent, so the allowance is three times
    the root-sum-square of those sizes over the set's near-zero coefficients."""
    from oracle import gauge as og
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    xp = og.apply_gauge(x, G) if G is not None else x
    _, _, _, U = sp.block_stats(xp, 16)                           # [L,2,B,H,nb,16,d]
    rms = np.sqrt((U * U).mean(axis=(-2, -1), keepdims=True))
    near = np.abs(U) <= rel_eps * rms
    c = 2.0 * lambda_r / (tau * n_blocks_total * 16 * d)
    W = np.einsum("ut,...tc->...uc", sp.dct_matrix(16), sp.blocks(x, 16))  # [..., nb, 16, d]
    R = d // 16
    Wr2 = (W.reshape(W.shape[:-1] + (R, 16)) ** 2).sum(-1)       # [..., nb, 16, R]
    Cd2 = (sp.dct_matrix(d).reshape(d, R, 16) ** 2).sum(-1)     # [d, R]
    size2 = c * c * np.einsum("...ur,vr->...uv", Wr2, Cd2)       # [..., nb, 16, d]
    tot2 = (near * size2).sum(axis=(-3, -2, -1))                 # [L, 2, B, H]
    return 3.0 * np.sqrt(tot2.sum(axis=2))                       # [L, 2, H] (summed over the batch)


@pytest.mark.parametrize("want_grad,T", [(False, 256), (True, 256), (True, 384)])
def test_stats_bf16_cache_with_gauge(want_grad, T):
    """T = 256: two 128-token tiles per head slice, so the dL/dG kernel's work unit
    is half a slice (two partials per slice); T = 384: an odd tile count, one unit
    of three tiles per slice."""
    need_gpu()
    L, B, H, d = 2, 2, 2, 128
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
    """One 4096-token window of the 8B-shaped cache with the gradient through a g = 16
    gauge on the bf16 cache (the launch the benchmark times: 512 head slices over 148
    CTAs, several slices per CTA): totals, and on sampled (l, s, h) slices the per-block
    values and that gauge set's dL/dG against the oracle: the frequency term alone
    (lambda_r = 0) within 1e-4 Frobenius-relative, the full objective within 1e-4 plus
    the rate kink's allowance."""
    need_gpu()
    L, B, H, T, d = 32, 1, 8, 4096, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=3, device="cuda", n_outliers=4)
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=3))
    lf, lr, tot, dG = run_stats(kv, G, True, False)
    _, _, _, dG_f = run_stats(kv, G, True, False, lambda_r=0.0)
    lf0, lr0, tot0, _ = run_stats(kv, G, False, False)  # statistics only: the tile-balanced kernel
    # oracle on a few (l, s, h) slices: per-block values, and dG of those gauge sets
    dG = dG.reshape(L, 2, H, 8, 16, 16)
    dG_f = dG_f.reshape(L, 2, H, 8, 16, 16)
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
        assert np.all(np.abs(lf0[base:base + nb] - rl) <= 1e-4 * np.maximum(np.abs(rl), 1e-3))
        assert np.all(np.abs(lr0[base:base + nb] - rr) <= 1e-4 * np.maximum(np.abs(rr), 1e-3))
        # dG of this gauge set is this slice's partial (B = 1).  The oracle's one-slice call
        # normalizes by its own block count; the window's objective by all blocks of the window,
        # and every term of dL/dG carries 1 / n_blocks, so the slice's share is scaled by
        # nb / n_total.  With the rate term the difference may include the sign decisions at
        # its kink (rate_kink_allowance); the frequency term alone must match within 1e-4.
        scale = nb / (L * 2 * B * H * nb)
        ref_g = sp.spectral_stats(x, Gs, want_grad=True)["dG"][0, 0, 0] * scale
        allow = rate_kink_allowance(x, Gs, L * 2 * B * H * nb)[0, 0, 0]
        err = np.sqrt(((dG[l, s, h].astype(np.float64) - ref_g) ** 2).sum())
        assert err <= 1e-4 * np.sqrt((ref_g ** 2).sum()) + allow, "dG of gauge set %s: %.3g (allowance %.3g)" % (
            (l, s, h), err / np.sqrt((ref_g ** 2).sum()), allow / np.sqrt((ref_g ** 2).sum()))
        ref_f = sp.spectral_stats(x, Gs, want_grad=True, lambda_r=0.0)["dG"][0, 0, 0] * scale
        got_f = dG_f[l, s, h].astype(np.float64)
        rel = np.sqrt(((got_f - ref_f) ** 2).sum() / (ref_f ** 2).sum())
        assert rel <= 1e-4, "frequency-term dG of gauge set %s: %.3g" % ((l, s, h), rel)
    assert tot[2] == L * 2 * B * H * nb
    lam_r = float(np.float32(0.02))  # lambda_r crosses the C ABI as fp32
    assert abs(tot[3] - (tot[0] / tot[2] + lam_r * tot[1] / tot[2])) <= 1e-12 * abs(tot[3])
    assert np.isfinite(dG).all()
    assert np.all(np.abs(tot0 - tot) <= 1e-5 * np.abs(tot))


@pytest.mark.parametrize("gauged", [True, False])
def test_stats_forward_tile_ranges(gauged):
    """Statistics without dL/dG split the 128-token tiles of all head slices into
    contiguous ranges, one per CTA: 4 x 2 x 1 x 4 slices of 2048 tokens are 512 tiles
    over at most 148 CTAs, so ranges start inside a slice, cross slice boundaries
    (each with its own gauge) and wrap the 4-stage ring.  Every block against the
    oracle, with a g = 16 gauge and without one."""
    need_gpu()
    L, B, H, T, d = 4, 1, 4, 2048, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=8, device="cuda", n_outliers=4)
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=8)) if gauged else None
    lf, lr, tot, _ = run_stats(kv, G, False, False)
    Gn = G.cpu().numpy().astype(np.float64) if gauged else None
    ref = sp.spectral_stats(bf16_np(kv), Gn)
    _check(ref, lf, lr, tot)


@pytest.mark.parametrize("L,H,T", [(8, 8, 128), (4, 8, 256), (4, 4, 384)])
def test_stats_forward_short_slices(L, H, T):
    """Statistics only, with a gauge, on slices of one, two and three 128-token tiles:
    fewer tiles than the forward kernel's four token parts, whose turns at building
    the next slice's M then fall on the slice's first tile in the CTA's range.  256,
    256 and 192 tiles over at most 148 CTAs, so ranges of one or two tiles cross slice
    boundaries.  Every block against the oracle."""
    need_gpu()
    B, d = 2, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=9, device="cuda", n_outliers=2)
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=9))
    lf, lr, tot, _ = run_stats(kv, G, False, False)
    ref = sp.spectral_stats(bf16_np(kv), G.cpu().numpy().astype(np.float64))
    _check(ref, lf, lr, tot)


@pytest.mark.parametrize("want_grad", [False, True])
def test_stats_large_magnitudes(want_grad):
    """The rate sum takes log2 of products of four arguments 1 + |U| / tau; a product
    overflows once |U| / tau passes about 2^32 and that block's sum is taken again two
    arguments at a time.  A head slice at 1e9 (every block overflows), a channel at 3e8
    (some coefficients of every block of its slice), a block at 1e7 (near the limit)
    and ordinary blocks beside them, against the oracle."""
    need_gpu()
    L, B, H, T, d = 2, 1, 2, 512, 128
    g = torch.Generator().manual_seed(33)
    x = torch.randn((L, 2, B, H, T, d), generator=g)
    x[0, 0, 0, 1] *= 1e9
    x[1, 1, 0, 0, :, 5] *= 3e8
    x[1, 0, 0, 1, 64:80] *= 1e7
    x = x.to(torch.bfloat16).cuda().contiguous()
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=33))
    lf, lr, tot, _ = run_stats(x, G, want_grad, False)
    ref = sp.spectral_stats(bf16_np(x), G.cpu().numpy().astype(np.float64))
    _check(ref, lf, lr, tot)


@pytest.mark.parametrize("gauged", [True, False])
def test_stats_fp32_input_tile_ranges(gauged):
    """fp32 input (already gauged, or with a g = 16 gauge applied in the kernel) takes the
    tensor-core statistics kernel too: each tile is split into bf16 hi + lo in shared
    memory and the channel GEMM runs three terms.  512 tiles of 4 x 2 x 1 x 4 slices of
    2048 tokens over at most 148 CTAs: ranges cross slices and wrap the 2-stage fp32 ring.
    Values span a wide range (N(0, 3) with 100x outlier channels and a 1e-3 scaled head),
    every block against the oracle."""
    need_gpu()
    L, B, H, T, d = 4, 1, 4, 2048, 128
    g = torch.Generator().manual_seed(21)
    x = torch.randn((L, 2, B, H, T, d), generator=g) * 3
    x[..., [7, 90]] *= 100.0
    x[:, :, :, 3] *= 1e-3
    x[0, 0, 0, 1, 16:32] = 0.0          # an all-zero block
    x = x.cuda().contiguous()
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=21)) if gauged else None
    lf, lr, tot, _ = run_stats(x, G, False, True)
    Gn = G.cpu().numpy().astype(np.float64) if gauged else None
    ref = sp.spectral_stats(x.cpu().numpy().astype(np.float64), Gn)
    _check(ref, lf, lr, tot)


@pytest.mark.parametrize("want_grad", [False, True])
def test_stats_tiny_config_d64(want_grad):
    """The small reference cache (1 x 2 x 1 x 2 x 1024 x 64, g = 16): the statistic spans
    the whole 64-channel head (r_uv with d - 1 = 63), CUDA-core kernel."""
    need_gpu()
    L, B, H, T, d = 1, 1, 2, 1024, 64
    kv = synth.kv_cache(L, B, H, T, d, seed=9, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, d // 16, 16, sigma=0.1, seed=9))
    lf, lr, tot, dG = run_stats(kv, G, want_grad, False)
    ref = sp.spectral_stats(bf16_np(kv), G.cpu().numpy().astype(np.float64), want_grad=want_grad)
    _check(ref, lf, lr, tot, dG)


def test_stats_d64_fp32_and_degenerate_blocks():
    need_gpu()
    L, B, H, T, d = 2, 2, 1, 96, 64
    g = torch.Generator().manual_seed(6)
    x = (torch.randn((L, 2, B, H, T, d), generator=g) * 2).cuda()
    x[1, 0, 1, 0, 16:32] = 0.0          # all-zero block
    x[0, 1, 0, 0, 48:64] = -0.75        # constant block
    lf, lr, tot, _ = run_stats(x, None, False, True)
    ref = sp.spectral_stats(x.cpu().numpy().astype(np.float64), None)
    _check(ref, lf, lr, tot)


@pytest.mark.parametrize("want_grad", [False, True])
def test_stats_d128_ragged_token_count(want_grad):
    """d = 128 with T = 96 (not a multiple of the tensor-core kernel's 128-token tile):
    the CUDA-core kernel, with B = 3 (dG summed over the batch in order)."""
    need_gpu()
    L, B, H, T, d = 1, 3, 2, 96, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=12, device="cuda")
    G = oracle_gauge(synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=12))
    lf, lr, tot, dG = run_stats(kv, G, want_grad, False)
    ref = sp.spectral_stats(bf16_np(kv), G.cpu().numpy().astype(np.float64), want_grad=want_grad)
    _check(ref, lf, lr, tot, dG)
