"""Pins of the oracle's spectral statistics: brute-force and library DCT,
closed forms of L_freq / L_rate, Parseval, gauge invariance of the energy, and
finite differences for the gradients."""
import numpy as np
import pytest
import scipy.fft

from oracle import gauge as og
from oracle import spectral as sp


def _dct2_brute(X):
    """Direct double sum of the orthonormal 2-D DCT-II."""
    N, M = X.shape
    U = np.zeros((N, M))
    for u in range(N):
        for v in range(M):
            au = np.sqrt((1.0 if u == 0 else 2.0) / N)
            av = np.sqrt((1.0 if v == 0 else 2.0) / M)
            acc = 0.0
            for n in range(N):
                for m in range(M):
                    acc += X[n, m] * np.cos(np.pi * (2 * n + 1) * u / (2 * N)) * np.cos(np.pi * (2 * m + 1) * v / (2 * M))
            U[u, v] = au * av * acc
    return U


@pytest.mark.parametrize("shape", [(4, 4), (4, 8), (16, 8)])
def test_dct_brute_force(shape):
    X = np.random.default_rng(0).standard_normal(shape)
    assert np.abs(sp.dct2_blocks(X[None]) [0] - _dct2_brute(X)).max() < 1e-13


def test_dct_against_library_16x128():
    X = np.random.default_rng(1).standard_normal((3, 16, 128))
    want = scipy.fft.dctn(X, type=2, norm="ortho", axes=(-2, -1))
    assert np.abs(sp.dct2_blocks(X) - want).max() < 1e-12


@pytest.mark.parametrize("n", [4, 16, 64, 128])
def test_dct_orthonormal(n):
    C = sp.dct_matrix(n)
    assert np.abs(C @ C.T - np.eye(n)).max() < 1e-13


def test_radius_corners():
    r = sp.radius(16, 128)
    assert r[0, 0] == 0.0 and abs(r[15, 127] - 1.0) < 1e-15
    assert abs(r[15, 0] - 1 / np.sqrt(2)) < 1e-15 and abs(r[0, 127] - 1 / np.sqrt(2)) < 1e-15


def test_constant_block_has_zero_centroid():
    x = np.full((16, 128), 2.5)
    lf, lr, E, U = sp.block_stats(x, 16)
    assert abs(lf[0]) < 1e-15
    assert abs(U[0, 0, 0] - 2.5 * np.sqrt(16 * 128)) < 1e-11
    assert np.abs(U[0]).sum() - abs(U[0, 0, 0]) < 1e-10


@pytest.mark.parametrize("u,v", [(0, 0), (1, 0), (0, 5), (7, 64), (15, 127)])
def test_basis_function_centroid_is_its_radius(u, v):
    Ct, Cd = sp.dct_matrix(16), sp.dct_matrix(128)
    X = np.outer(Ct[u], Cd[v])                # inverse DCT of a unit coefficient at (u, v)
    lf, lr, E, U = sp.block_stats(X, 16)
    assert abs(lf[0] - sp.radius(16, 128)[u, v]) < 1e-12
    assert abs(E[0] - 1.0) < 1e-12
    # single coefficient a = 1: L_rate = log(1 + 1/tau) / N (other U are ~1e-16)
    assert abs(lr[0] - np.log1p(1.0 / sp.TAU) / (16 * 128)) < 1e-10


def test_zero_block():
    lf, lr, E, U = sp.block_stats(np.zeros((2, 32, 16)), 16)
    assert np.all(lf == 0) and np.all(lr == 0)


def test_parseval_and_gauge_invariant_energy():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 2, 1, 2, 64, 32))
    G = og.gauge_from_A(rng.normal(0, 0.3, (1, 2, 2, 2, 16, 16)))
    _, _, E0, _ = sp.block_stats(x, 16)
    _, _, E1, _ = sp.block_stats(og.apply_gauge(x, G), 16)
    xb = sp.blocks(x, 16)
    assert np.abs(E0 - (xb ** 2).sum(axis=(-2, -1))).max() < 1e-11
    assert np.abs(E1 - E0).max() < 1e-11


def test_totals_and_objective():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 2, 1, 1, 48, 16))
    out = sp.spectral_stats(x, None, tb=16)
    t = out["totals"]
    assert t[2] == 6
    assert abs(t[3] - (t[0] / 6 + 0.02 * t[1] / 6)) < 1e-15
    assert abs(t[0] / 6 - out["lfreq"].mean()) < 1e-15


def _objective(x, G):
    return sp.spectral_stats(x, G, tb=16)["totals"][3]


def test_grad_G_finite_differences():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, 2, 1, 1, 32, 16))
    x[0, 0, 0, 0, 16:] = 1.0                        # a nearly constant block
    G = og.gauge_from_A(rng.normal(0, 0.3, (1, 2, 1, 2, 8, 8)))
    dG = sp.spectral_stats(x, G, tb=16, want_grad=True)["dG"]
    h = 1e-6
    for idx in [(0, 0, 0, 0, 1, 2), (0, 1, 0, 1, 7, 0), (0, 0, 0, 1, 3, 3), (0, 1, 0, 0, 0, 5)]:
        Gp, Gm = G.copy(), G.copy()
        Gp[idx] += h
        Gm[idx] -= h
        fd = (_objective(x, Gp) - _objective(x, Gm)) / (2 * h)
        assert abs(fd - dG[idx]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9


def test_grad_A_finite_differences_and_antisymmetry():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 2, 1, 1, 32, 16))
    A = rng.normal(0, 0.3, (1, 2, 1, 2, 8, 8))
    G = og.gauge_from_A(A)
    dG = sp.spectral_stats(x, G, tb=16, want_grad=True)["dG"]
    dA = sp.grad_A(A, dG)
    assert np.abs(dA + np.swapaxes(dA, -1, -2)).max() < 1e-14
    h = 1e-6
    for idx in [(0, 0, 0, 0, 1, 2), (0, 1, 0, 1, 6, 3), (0, 0, 0, 1, 0, 7)]:
        Ap, Am = A.copy(), A.copy()
        Ap[idx] += h
        Am[idx] -= h
        fd = (_objective(x, og.gauge_from_A(Ap)) - _objective(x, og.gauge_from_A(Am))) / (2 * h)
        assert abs(fd - dA[idx]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9


def test_frechet_identity_at_zero():
    E = np.random.default_rng(6).standard_normal((5, 5))
    assert np.abs(sp.frechet_exp(np.zeros((5, 5)), E) - E).max() < 1e-14
