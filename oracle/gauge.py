"""The cache-coordinate gauge (test infrastructure only).

Codec-Gauge, Problem statement and overview (channel groups): for layer l,
cache type s in {K, V}, head h and channel group r the head dimension d splits
into R = d / g groups of g channels; X[b, h, t, r] is the g-vector of one token
in one group, and one invertible gauge G_{l,s,h,r} acts on it.  It mixes
channels inside a group only, never tokens, heads or layers.

Codec-Gauge, Method (gauge parameterization): G = exp(A - A^T); A - A^T is
skew-symmetric, so G is orthogonal and G^{-1} = G^T.  (The displayed formula is
missing from the page; its text names exp(.) and the skew matrix A - A^T.)

Array conventions used by the whole oracle:
  kv : [L, 2, B, H, T, d]   (s = 0 keys, s = 1 values)
  A, G : [L, 2, H, R, g, g] (one gauge per layer, K/V, head and group; shared
                             over the batch)
  y[..., t, r*g + i] = sum_j G[r, i, j] * x[..., t, r*g + j]
"""
import math
import numpy as np

from .fpround import fma_f32, fl32, fl_bf16


def skew(A):
    """S = A - A^T over the last two axes."""
    A = np.asarray(A, dtype=np.float64)
    return A - np.swapaxes(A, -1, -2)


def _norm1(M):
    return np.abs(M).sum(axis=-2).max()


def expm_taylor(S, degree=18):
    """exp(S) for one square matrix by scaling and squaring with a Taylor core.

    Scaling and squaring (Higham, "The scaling and squaring method for the
    matrix exponential revisited", 2005): pick s with ||S / 2^s||_1 <= 1/2, sum
    the Taylor series of exp(S / 2^s) to ``degree`` (truncation error below
    (1/2)^19 / 19! ~ 2e-23 relative), then square s times.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    nrm = _norm1(S)
    s = 0 if nrm == 0 else max(0, int(math.ceil(math.log2(nrm))) + 1)
    M = S / (2.0 ** s)
    I = np.eye(n)
    E = I.copy()
    for k in range(degree, 0, -1):  # Horner: I + M/1 (I + M/2 (I + ...))
        E = I + (M @ E) / k
    for _ in range(s):
        E = E @ E
    return E


_PADE13_B = (64764752532480000.0, 32382376266240000.0, 7771770303897600.0,
             1187353796428800.0, 129060195264000.0, 10559470521600.0,
             670442572800.0, 33522128640.0, 1323241920.0, 40840800.0,
             960960.0, 16380.0, 182.0, 1.0)


def expm_pade13(S):
    """exp(S) by the [13/13] Pade approximant with scaling and squaring.

    Higham 2005 (same paper): theta_13 = 5.371920351148152 bounds the scaled
    norm; the numerator and denominator share even and odd parts U, V built
    from S^2, S^4, S^6, and r_13 = (V - U)^{-1} (V + U).  Used only to cross-
    check ``expm_taylor``.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    nrm = _norm1(S)
    theta = 5.371920351148152
    s = 0 if nrm <= theta else int(math.ceil(math.log2(nrm / theta)))
    M = S / (2.0 ** s)
    b = _PADE13_B
    I = np.eye(n)
    M2 = M @ M
    M4 = M2 @ M2
    M6 = M4 @ M2
    U = M @ (M6 @ (b[13] * M6 + b[11] * M4 + b[9] * M2)
             + b[7] * M6 + b[5] * M4 + b[3] * M2 + b[1] * I)
    V = (M6 @ (b[12] * M6 + b[10] * M4 + b[8] * M2)
         + b[6] * M6 + b[4] * M4 + b[2] * M2 + b[0] * I)
    E = np.linalg.solve(V - U, V + U)
    for _ in range(s):
        E = E @ E
    return E


def gauge_from_A(A):
    """G = exp(A - A^T) for every trailing g x g matrix of A (fp64)."""
    A = np.asarray(A, dtype=np.float64)
    flat = A.reshape(-1, A.shape[-2], A.shape[-1])
    out = np.stack([expm_taylor(skew(a)) for a in flat])
    return out.reshape(A.shape)


def _grouped(x, g):
    """View [..., T, d] as [..., T, R, g]."""
    return x.reshape(x.shape[:-1] + (x.shape[-1] // g, g))


def apply_gauge(kv, G):
    """Exact gauge y = G x per token and group, in fp64.

    kv [L, 2, B, H, T, d]; G [L, 2, H, R, g, g].  Returns y with kv's shape.
    """
    kv = np.asarray(kv, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    g = G.shape[-1]
    xg = _grouped(kv, g)                       # [L,2,B,H,T,R,g]
    y = np.einsum("lshrij,lsbhtrj->lsbhtri", G, xg)
    return y.reshape(kv.shape)


def apply_inverse_gauge(y, G):
    """Exact inverse gauge x = G^T y per token and group, in fp64."""
    y = np.asarray(y, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    g = G.shape[-1]
    yg = _grouped(y, g)
    x = np.einsum("lshrji,lsbhtrj->lsbhtri", G, yg)
    return x.reshape(y.shape)


def apply_gauge_f32_chain(kv, G32):
    """The encoder's gauged values: fp32 FMA chain in channel-index order.

    The quantizer turns floating-point values into integer codes, so the codes
    are only reproducible if the values it sees are.  The codec therefore fixes
    the fp32 arithmetic of y = G x: for every output i,
        acc = +0;  for j = 0 .. g-1:  acc = fl32(G[i, j] * x[j] + acc)  (fused)
    and y_i = acc.  This is the plain dot product in index order, with one
    IEEE fp32 fused multiply-add per term.  G32 must hold float32 values, kv
    bf16 values (both exact in float32).
    """
    kv = np.asarray(kv, dtype=np.float64)
    G32 = np.asarray(G32, dtype=np.float64)
    g = G32.shape[-1]
    xg = _grouped(kv, g)                       # [L,2,B,H,T,R,g]
    L, S2, B, H, T, R, _ = xg.shape
    # broadcast G over batch and tokens: Gb[l,s,1,h,1,r,i,j]
    Gb = G32[:, :, None, :, None, :, :, :]
    acc = np.zeros((L, S2, B, H, T, R, g), dtype=np.float64)
    for j in range(g):
        acc = fma_f32(Gb[..., :, j], xg[..., None, j], acc)
    return acc.reshape(kv.shape)


def round_gauge_bf16(G):
    """bf16 (RNE) copy of an fp32 gauge, as used by the full-head contraction."""
    return fl_bf16(fl32(G))
