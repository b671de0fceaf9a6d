"""Gauge training step (test infrastructure only).

Codec-Gauge, Method (gauge training): the gauge parameters are optimized with
AdamW over 4096-token windows on L = lambda_f mean L_freq + lambda_r mean L_rate
(T_b = 16, lambda_f = 1.0, lambda_r = 0.02, tau = 0.04).  The pages give no
optimizer settings; the reading taken is torch's AdamW defaults (lr 1e-3,
betas 0.9 / 0.999, eps 1e-8, weight decay 0.01), one step per window.

AdamW: Loshchilov & Hutter, "Decoupled weight decay regularization" (2019),
Algorithm 2, with bias-corrected moments:
    m_t = b1 m_{t-1} + (1 - b1) g_t
    v_t = b2 v_{t-1} + (1 - b2) g_t^2
    p_t = p_{t-1} - lr (m_t / (1 - b1^t) / (sqrt(v_t / (1 - b2^t)) + eps) + wd p_{t-1})
"""
import numpy as np

from . import gauge as _g
from . import spectral as _sp

ADAMW_DEFAULTS = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def adamw_step(p, grad, m, v, t, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01):
    """One AdamW step in fp64; returns (p, m, v) (new arrays).  t is 1-based."""
    p = np.asarray(p, np.float64)
    grad = np.asarray(grad, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * grad
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * grad * grad
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    return p - lr * (mhat / (np.sqrt(vhat) + eps) + weight_decay * p), m, v


def train_step(A, kv, m, v, t, lambda_f=1.0, lambda_r=0.02, tau=0.04, **adamw):
    """One optimizer step on one window kv [L, 2, B, H, T, d]: returns
    (A, m, v, totals) with the window's totals before the update."""
    A = np.asarray(A, np.float64)
    G = _g.gauge_from_A(A)
    out = _sp.spectral_stats(kv, G, tau=tau, lambda_f=lambda_f, lambda_r=lambda_r, want_grad=True)
    dA = _sp.grad_A(A, out["dG"])
    hp = dict(ADAMW_DEFAULTS)
    hp.update(adamw)
    A2, m2, v2 = adamw_step(A, dA, m, v, t, **hp)
    return A2, m2, v2, out["totals"]
