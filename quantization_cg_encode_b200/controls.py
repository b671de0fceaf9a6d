"""Coordinate-control gauges beside the learned one (Codec-Gauge, Experimental
setup and Results: identity, random orthogonal, Hadamard, DCT and PCA/KLT
controls run through the same backend at the same rate).

Identity, random orthogonal (Haar) and DCT-II gauges are in ``synth``.  This
module adds the normalized Sylvester-Hadamard gauge and the PCA/KLT gauge,
whose basis is the uncentered second-moment eigenbasis of each (layer, K/V,
head, group): the Gram matrices are summed on the GPU by ``cg_group_gram`` and
the symmetric eigensolver runs on the host (a one-time set-up step, like the
gauge training itself).
"""
import math

import numpy as np
import torch

from . import cg


def hadamard_matrix(g):
    """Normalized Sylvester Hadamard matrix H_g / sqrt(g) (g a power of two):
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]; symmetric and orthogonal."""
    if g < 1 or g & (g - 1):
        raise ValueError("g must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < g:
        H = np.block([[H, H], [H, -H]])
    return H / math.sqrt(g)


def hadamard_gauge(L, H, R, g, device="cpu"):
    """fp32 [L, 2, H, R, g, g], the same Hadamard matrix for every group."""
    M = torch.from_numpy(hadamard_matrix(g)).float()
    return M.expand(L, 2, H, R, g, g).contiguous().to(device)


def klt_from_gram(gram):
    """PCA/KLT gauge from Gram matrices [..., g, g] (fp64): the rows of G are the
    eigenvectors of C in order of decreasing eigenvalue, so y = G x has
    uncorrelated second moments sorted by energy.  Each row's sign is fixed so
    that its entry of largest magnitude is positive.  Returns fp32."""
    C = np.asarray(gram, np.float64)
    C = 0.5 * (C + np.swapaxes(C, -1, -2))
    w, V = np.linalg.eigh(C)                        # ascending eigenvalues, eigenvectors in columns
    V = V[..., ::-1]                                # descending
    G = np.swapaxes(V, -1, -2).copy()               # rows = eigenvectors
    idx = np.argmax(np.abs(G), axis=-1)
    sgn = np.sign(np.take_along_axis(G, idx[..., None], axis=-1))
    sgn[sgn == 0] = 1.0
    return (G * sgn).astype(np.float32)


def klt_gauge(kv, g, t0=0, nt=None, stream=None):
    """PCA/KLT gauge [L, 2, H, d/g, g, g] (fp32, on kv's device) of a bf16 cache
    [L, 2, B, H, T, d]: GPU Gram matrices, host eigensolver."""
    kvd = cg.kv_desc_of(kv)
    gram = torch.empty((kvd.layers, 2, kvd.heads, kvd.d_head // g, g, g), dtype=torch.float64, device=kv.device)
    cg.cg_group_gram(kvd, g, kv, gram, t0, nt, stream=stream)
    return torch.from_numpy(klt_from_gram(gram.cpu().numpy())).to(kv.device)
