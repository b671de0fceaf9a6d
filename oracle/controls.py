"""Coordinate-control gauges (test infrastructure only).

Codec-Gauge, Experimental setup and Results: identity, random orthogonal,
Hadamard, DCT and PCA/KLT controls run through the same backend; PCA/KLT uses
the uncentered second-moment eigenbasis computed at the same layer, K/V, head
and group granularity.
"""
import numpy as np


def hadamard(g):
    """Normalized Sylvester Hadamard matrix: entries +-1/sqrt(g), H H^T = I."""
    assert g >= 1 and g & (g - 1) == 0
    H = np.array([[1.0]])
    while H.shape[0] < g:
        H = np.concatenate([np.concatenate([H, H], 1), np.concatenate([H, -H], 1)], 0)
    return H / np.sqrt(g)


def gram(kv, g, t0=0, nt=None):
    """C[l, s, h, r] = sum_{b, t} x x^T over the g-vectors of group r, tokens
    [t0, t0 + nt); kv [L, 2, B, H, T, d] -> [L, 2, H, d/g, g, g] (fp64)."""
    kv = np.asarray(kv, np.float64)
    L, S2, B, H, T, d = kv.shape
    nt = T - t0 if nt is None else nt
    x = kv[..., t0:t0 + nt, :].reshape(L, S2, B, H, nt, d // g, g)
    return np.einsum("lsbhtri,lsbhtrj->lshrij", x, x)


def klt(C):
    """Rows = eigenvectors of the symmetric C in order of decreasing eigenvalue
    (so G C G^T is diagonal, largest first); each row's largest-magnitude entry
    is made positive.  Returns (G, eigenvalues descending)."""
    C = np.asarray(C, np.float64)
    w, V = np.linalg.eigh(0.5 * (C + np.swapaxes(C, -1, -2)))
    w = w[..., ::-1]
    G = np.swapaxes(V[..., ::-1], -1, -2).copy()
    idx = np.argmax(np.abs(G), axis=-1)
    sgn = np.sign(np.take_along_axis(G, idx[..., None], axis=-1))
    sgn[sgn == 0] = 1.0
    return G * sgn, w
