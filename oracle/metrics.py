"""Cache-side metrics (test infrastructure only).

Codec-Gauge, Experimental setup (metrics): compressed bytes, actual bits/value
from the measured bytes, KV MSE, NRMSE and maximum absolute error.  The page
gives no NRMSE formula; the plainest reading is ||x - x_hat||_2 / ||x||_2.
"""
import numpy as np


def nrmse(x, xhat):
    x = np.asarray(x, np.float64)
    xhat = np.asarray(xhat, np.float64)
    den = np.sqrt((x * x).sum())
    return float(np.sqrt(((x - xhat) ** 2).sum()) / den) if den > 0 else 0.0


def mse(x, xhat):
    return float(((np.asarray(x, np.float64) - np.asarray(xhat, np.float64)) ** 2).mean())


def max_abs(x, xhat):
    return float(np.abs(np.asarray(x, np.float64) - np.asarray(xhat, np.float64)).max())


def bits_per_value(code_bytes, scale_count, n_values):
    """8 (code bytes + 2 bytes of fp16 scale + 2 of fp16 zero per range) / N_KV."""
    return 8.0 * (code_bytes + 4 * scale_count) / n_values
