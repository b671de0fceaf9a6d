"""Seeded synthetic inputs shaped like the KV caches the Codec-Gauge paper
measures on (it trains and evaluates on prefill KV tensors of real models,
which are not available here).  This module holds no codec arithmetic: it only
draws inputs, and both the CUDA library's tests and the CPU checker consume
the very same tensors.

Recipe (one generator for every cache shape):
  keys   : AR(1) along tokens, x_t = 0.9 x_{t-1} + e_t, e_t ~ N(0, 1), started
           from the stationary law N(0, 1 / (1 - 0.9^2)); then every channel of
           every (layer, head) is scaled by an independent lognormal(0, 0.5)
           factor, and the outlier channels by a further x10.
  values : AR(1) with rho = 0.5, unit scale, same start rule.
  outlier channels: an explicit list for every head (the 1-layer test cache uses
           channels 3 and 17), or n seeded distinct channels per (layer, head).
  gauge parameters A ~ N(0, sigma^2) i.i.d. per g x g matrix.
  control gauges: identity, Haar-random orthogonal (QR of a Gaussian matrix
           with the sign of diag(R) folded in, Mezzadri 2007), orthonormal
           DCT-II basis.
All tensors are torch tensors; the cache is bf16 in [L, 2, B, H, T, d] order.
"""
import math

import numpy as np
import torch


def _ar1_(out, rho, gen, chunk=512):
    """Fill out[..., T, d] (fp32) with a stationary AR(1) along T, in place."""
    *lead, T, d = out.shape
    dev = out.device
    x_prev = torch.randn(tuple(lead) + (d,), generator=gen, device=dev) / math.sqrt(1.0 - rho * rho)
    # x[t0 + k] = rho^(k+1) x_prev + sum_{m<=k} rho^(k-m) e[t0 + m]
    k = torch.arange(chunk, device=dev, dtype=torch.float64)
    M = torch.where(k[:, None] >= k[None, :], rho ** (k[:, None] - k[None, :]), torch.zeros((), dtype=torch.float64, device=dev)).float()
    p = (rho ** (k + 1)).float()
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        e = torch.randn(tuple(lead) + (n, d), generator=gen, device=dev)
        blk = torch.matmul(M[:n, :n], e) + p[:n, None] * x_prev[..., None, :]
        out[..., t0:t0 + n, :] = blk
        x_prev = blk[..., -1, :]
    return out


def kv_cache(L, B, H, T, d, seed=0, device="cpu", key_rho=0.9, value_rho=0.5,
             outlier_channels=(3, 17), n_outliers=None, scale_sigma=0.5, outlier_gain=10.0):
    """bf16 cache [L, 2, B, H, T, d] following the module recipe.

    ``n_outliers`` (if given) replaces ``outlier_channels`` by that many seeded
    distinct channels per (layer, head).  Generated layer by layer so the fp32
    working set stays small.
    """
    prev_tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        gen = torch.Generator(device=device).manual_seed(int(seed))
        out = torch.empty((L, 2, B, H, T, d), dtype=torch.bfloat16, device=device)
        cpu_gen = torch.Generator().manual_seed(int(seed) + 1)
        for l in range(L):
            k = torch.empty((B, H, T, d), dtype=torch.float32, device=device)
            _ar1_(k, key_rho, gen)
            scale = torch.exp(scale_sigma * torch.randn((H, d), generator=cpu_gen)).to(device)
            for h in range(H):
                if n_outliers is not None:
                    ch = torch.randperm(d, generator=cpu_gen)[:n_outliers].tolist()
                else:
                    ch = list(outlier_channels)
                for c in ch:
                    scale[h, c] *= outlier_gain
            k *= scale[None, :, None, :]
            out[l, 0] = k.to(torch.bfloat16)
            v = torch.empty((B, H, T, d), dtype=torch.float32, device=device)
            _ar1_(v, value_rho, gen)
            out[l, 1] = v.to(torch.bfloat16)
        return out
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev_tf32


def gauge_params(L, H, R, g, sigma=0.1, seed=0, device="cpu"):
    """A ~ N(0, sigma^2), fp32 [L, 2, H, R, g, g]."""
    gen = torch.Generator().manual_seed(int(seed) + 7)
    return (sigma * torch.randn((L, 2, H, R, g, g), generator=gen)).to(device)


def identity_gauge(L, H, R, g, device="cpu"):
    return torch.eye(g).expand(L, 2, H, R, g, g).contiguous().to(device)


def haar_gauge(L, H, R, g, seed=0, device="cpu"):
    """Haar-distributed orthogonal matrices, fp32 [L, 2, H, R, g, g]."""
    rng = np.random.default_rng(int(seed) + 11)
    Z = rng.standard_normal((L * 2 * H * R, g, g))
    out = np.empty_like(Z)
    for i, z in enumerate(Z):
        q, r = np.linalg.qr(z)
        out[i] = q * np.sign(np.diag(r))[None, :]
    return torch.from_numpy(out.reshape(L, 2, H, R, g, g)).float().to(device)


def dct_gauge(L, H, R, g, device="cpu"):
    """The orthonormal DCT-II basis as a fixed control gauge (rows = frequencies)."""
    n = np.arange(g, dtype=np.float64)
    rows = [np.cos(np.pi * (n + 0.5) * k / g) * (math.sqrt(1.0 / g) if k == 0 else math.sqrt(2.0 / g))
            for k in range(g)]
    C = torch.from_numpy(np.stack(rows)).float()
    return C.expand(L, 2, H, R, g, g).contiguous().to(device)
