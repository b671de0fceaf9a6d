"""Gauge training on the GPU (Codec-Gauge, Method: gauge training).

The gauge parameters A of every (layer, K/V, head, group) are optimized with
AdamW on L = lambda_f mean L_freq + lambda_r mean L_rate over 4096-token
windows of cached keys and values.  One step on one window:

    G  = exp(A - A^T)                          cg_gauge_build
    L, dL/dG                                   cg_spectral_stats (gradient on)
    dL/dA = L_exp(S^T, dG) - (...)^T           cg_gauge_grad
    A <- AdamW(A, dL/dA)                       cg_adamw_step

This module only sequences those library calls and keeps the buffers; all
arithmetic runs in the CUDA library.  Readings where the pages are silent:
one optimizer step per window (the window is the batch), torch's AdamW
defaults (lr 1e-3, betas 0.9 / 0.999, eps 1e-8, weight decay 0.01), and the
pages' lambda_f = 1.0, lambda_r = 0.02, tau = 0.04, T_b = 16.
"""
import torch

from . import cg


class GaugeTrainer:
    """AdamW training of the group gauges of a cache shape (L, B, H, T, d)."""

    def __init__(self, A, kv_shape, hp=None, lambda_f=1.0, lambda_r=0.02, tau=0.04, stream=None):
        L, _, B, H, T, d = kv_shape
        self.g = A.shape[-1]
        self.A = A.contiguous()
        self.G = torch.empty_like(self.A)
        self.dG = torch.empty_like(self.A)
        self.dA = torch.empty_like(self.A)
        self.m = torch.zeros_like(self.A)
        self.v = torch.zeros_like(self.A)
        self.hp = hp if hp is not None else cg.adamw_desc()
        self.kvd = cg.kv_desc(L, B, H, T, d)
        self.st = cg.StatsDesc(16, self.g, 0, lambda_f, lambda_r, tau)
        nblk = L * 2 * B * H * T // 16
        dev = A.device
        self.lf = torch.empty(nblk, dtype=torch.float32, device=dev)
        self.lr = torch.empty_like(self.lf)
        self.totals = torch.empty(4, dtype=torch.float64, device=dev)
        ws = cg.cg_spectral_workspace_size(self.kvd, self.st, True)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        self.stream = stream
        self.t = 0

    def gauge(self):
        """G = exp(A - A^T) of the current parameters."""
        cg.cg_gauge_build(self.A, self.G, stream=self.stream)
        return self.G

    def step(self, kv):
        """One AdamW step on one bf16 window [L, 2, B, H, T, d]; returns the window's
        fp64 totals [sum L_freq, sum L_rate, n_blocks, L] before the update (device)."""
        self.gauge()
        cg.cg_spectral_stats(self.kvd, self.st, kv, self.G, self.lf, self.lr, self.totals, self.dG, self.ws,
                             stream=self.stream)
        cg.cg_gauge_grad(self.A, self.dG, self.dA, stream=self.stream)
        self.t += 1
        cg.cg_adamw_step(self.A, self.dA, self.m, self.v, self.hp, self.t, stream=self.stream)
        return self.totals

    def epoch(self, windows):
        """One pass over the windows; returns (mean L, mean L_freq) over the epoch."""
        acc = torch.zeros(4, dtype=torch.float64, device=self.A.device)
        for kv in windows:
            acc += self.step(kv)
        n = float(len(windows))
        tot = acc.cpu().tolist()
        return tot[3] / n, tot[0] / tot[2]
