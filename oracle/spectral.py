"""Spectral training statistics of the gauge (test infrastructure only).

Codec-Gauge, Method (frequency-distribution objective).  For a gauged cache
tensor X' = G X the token axis is cut into blocks of T_b tokens and every
T_b x d token-channel block (d = full head, even when the gauge is grouped) gets
a two-dimensional orthonormal DCT, U.  The page's equations for the DCT, the
normalized radius, the spectral centroid, the rate proxy and the objective were
stripped; this module takes these readings:

  DCT     : orthonormal DCT-II (Ahmed et al. 1974), U = C_Tb X'_blk C_d^T,
            C_N[k, n] = a_k cos(pi (2n + 1) k / (2N)), a_0 = sqrt(1/N),
            a_k = sqrt(2/N); u indexes token frequency, v channel frequency.
  radius  : r_uv = sqrt((u/(T_b-1))^2 + (v/(d-1))^2) / sqrt(2), in [0, 1].
  centroid: per block L_freq = sum r E / sum E with E_uv = U_uv^2 (the energy
            is defined in the page's text); a block with sum E = 0 gets 0.
  rate    : per block L_rate = mean log(1 + |U| / tau), tau = 0.04.  The page
            names a smooth, concave log-amplitude proxy with tau = 0.04; the
            formula itself is truncated, so this form is an assumption.
  totals  : unweighted means over blocks (all blocks have the same size);
            L = lambda_f mean(L_freq) + lambda_r mean(L_rate), lambda_f = 1.0,
            lambda_r = 0.02 (Method, training hyperparameters).
  concentration = 1 - L_freq (the quantity the paper tracks).

Parity status: pinned to these formulas (closed forms, Parseval, brute-force
DCT, finite differences); whether they equal the pages' elided equations is
"parity unpinned".
"""
import numpy as np

from .gauge import apply_gauge, expm_taylor, skew

TAU = 0.04
LAMBDA_F = 1.0
LAMBDA_R = 0.02


def dct_matrix(N):
    """Orthonormal DCT-II matrix C[k, n]."""
    k = np.arange(N)[:, None].astype(np.float64)
    n = np.arange(N)[None, :].astype(np.float64)
    C = np.cos(np.pi * (2.0 * n + 1.0) * k / (2.0 * N))
    C *= np.sqrt(2.0 / N)
    C[0, :] = np.sqrt(1.0 / N)
    return C


def radius(tb, d):
    u = np.arange(tb, dtype=np.float64)[:, None] / (tb - 1)
    v = np.arange(d, dtype=np.float64)[None, :] / (d - 1)
    return np.sqrt(u * u + v * v) / np.sqrt(2.0)


def blocks(xp, tb):
    """[..., T, d] -> [..., T/tb, tb, d]."""
    *lead, T, d = xp.shape
    return np.asarray(xp, np.float64).reshape(tuple(lead) + (T // tb, tb, d))


def dct2_blocks(xb):
    """U = C_tb X C_d^T for every trailing [tb, d] block."""
    tb, d = xb.shape[-2:]
    Ct, Cd = dct_matrix(tb), dct_matrix(d)
    return np.einsum("uk,...kn,vn->...uv", Ct, xb, Cd)


def block_stats(xp, tb=16, tau=TAU):
    """Per-block (L_freq, L_rate, E, U) of the gauged tensor xp [..., T, d]."""
    U = dct2_blocks(blocks(xp, tb))
    r = radius(tb, xp.shape[-1])
    E2 = U * U
    E = E2.sum(axis=(-2, -1))
    F = (r * E2).sum(axis=(-2, -1))
    lfreq = np.where(E > 0, F / np.where(E > 0, E, 1.0), 0.0)
    lrate = np.log1p(np.abs(U) / tau).mean(axis=(-2, -1))
    return lfreq, lrate, E, U


def totals(lfreq, lrate, lambda_f=LAMBDA_F, lambda_r=LAMBDA_R):
    """[sum L_freq, sum L_rate, n_blocks, L] over all blocks."""
    n = float(np.size(lfreq))
    sf = float(np.sum(lfreq))
    sr = float(np.sum(lrate))
    return np.array([sf, sr, n, lambda_f * sf / n + lambda_r * sr / n])


def grad_U(U, lfreq, E, n_blocks, tau=TAU, lambda_f=LAMBDA_F, lambda_r=LAMBDA_R):
    """dL/dU for L = lambda_f mean_blk L_freq + lambda_r mean_all log(1+|U|/tau).

    d L_freq,blk / dU_uv = 2 U_uv (r_uv - L_freq,blk) / E_blk  (0 when E_blk = 0)
    d log(1 + |U|/tau) / dU = sign(U) / (tau + |U|)           (sign(0) = 0)
    """
    tb, d = U.shape[-2:]
    r = radius(tb, d)
    n_coeff = n_blocks * tb * d
    Es = np.where(E > 0, E, 1.0)[..., None, None]
    gf = np.where((E > 0)[..., None, None], 2.0 * U * (r - lfreq[..., None, None]) / Es, 0.0)
    gr = np.sign(U) / (tau + np.abs(U))
    return lambda_f * gf / n_blocks + lambda_r * gr / n_coeff


def grad_xp(dU):
    """dL/dX' per block: C_tb^T dU C_d, returned as [..., T, d]."""
    tb, d = dU.shape[-2:]
    Ct, Cd = dct_matrix(tb), dct_matrix(d)
    dxb = np.einsum("uk,...uv,vn->...kn", Ct, dU, Cd)
    *lead, nb, _, _ = dxb.shape
    return dxb.reshape(tuple(lead) + (nb * tb, d))


def grad_G(dxp, kv, g):
    """dG[l,s,h,r,i,j] = sum_{b,t} dX'[l,s,b,h,t,r g+i] X[l,s,b,h,t,r g+j]."""
    L, S2, B, H, T, d = kv.shape
    R = d // g
    dx = np.asarray(dxp, np.float64).reshape(L, S2, B, H, T, R, g)
    x = np.asarray(kv, np.float64).reshape(L, S2, B, H, T, R, g)
    return np.einsum("lsbhtri,lsbhtrj->lshrij", dx, x)


def spectral_stats(kv, G=None, tb=16, tau=TAU, lambda_f=LAMBDA_F, lambda_r=LAMBDA_R,
                   want_grad=False):
    """Forward statistics (and dG when G is given and want_grad).

    kv [L, 2, B, H, T, d]: the gauged tensor when G is None, else the ungauged
    cache, gauged here in fp64 (X' = G X).  Returns dict with per-block
    lfreq/lrate [L, 2, B, H, T/tb], totals [4], and dG [L, 2, H, R, g, g].
    """
    kv = np.asarray(kv, np.float64)
    xp = kv if G is None else apply_gauge(kv, G)
    lfreq, lrate, E, U = block_stats(xp, tb, tau)
    out = dict(lfreq=lfreq, lrate=lrate, totals=totals(lfreq, lrate, lambda_f, lambda_r))
    if want_grad and G is not None:
        dU = grad_U(U, lfreq, E, lfreq.size, tau, lambda_f, lambda_r)
        out["dG"] = grad_G(grad_xp(dU), kv, G.shape[-1])
    return out


def frechet_exp(X, E):
    """Frechet derivative L_exp(X, E): upper-right block of exp([[X, E], [0, X]]).

    Van Loan 1978; Higham, Functions of Matrices 2008, section 10.
    """
    n = X.shape[0]
    M = np.zeros((2 * n, 2 * n))
    M[:n, :n] = X
    M[n:, n:] = X
    M[:n, n:] = E
    return expm_taylor(M)[:n, n:]


def grad_A(A, dG):
    """dL/dA from dL/dG for G = exp(A - A^T).

    The adjoint of E -> L_exp(S, E) is F -> L_exp(S^T, F), so dL/dS =
    L_exp(S^T, dG); S = A - A^T gives dL/dA = dS - dS^T.
    """
    A = np.asarray(A, np.float64)
    dG = np.asarray(dG, np.float64)
    flat_a = A.reshape(-1, A.shape[-2], A.shape[-1])
    flat_g = dG.reshape(flat_a.shape)
    out = []
    for a, gg in zip(flat_a, flat_g):
        S = skew(a)
        dS = frechet_exp(S.T, gg)
        out.append(dS - dS.T)
    return np.stack(out).reshape(A.shape)
