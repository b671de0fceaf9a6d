"""Pins of the oracle's gauge: closed forms, group structure, orthogonality,
an independent library expm, and exact rational arithmetic for the fp32 chain."""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

from oracle import gauge as og
from oracle.fpround import fl32, fl_bf16
from tests.test_oracle_fpround import _round_f32_exact


def test_expm_2x2_rotation_closed_form():
    for th in [0.0, 0.3, -1.7, 2.9]:
        S = np.array([[0.0, th], [-th, 0.0]])
        want = np.array([[np.cos(th), np.sin(th)], [-np.sin(th), np.cos(th)]])
        assert np.abs(og.expm_taylor(S) - want).max() < 1e-14
        assert np.abs(og.expm_pade13(S) - want).max() < 1e-14


def test_expm_block_diagonal_is_blockwise():
    rng = np.random.default_rng(0)
    S1, S2 = og.skew(rng.normal(0, 0.4, (3, 3))), og.skew(rng.normal(0, 0.4, (5, 5)))
    S = scipy.linalg.block_diag(S1, S2)
    E = og.expm_taylor(S)
    assert np.abs(E[:3, :3] - og.expm_taylor(S1)).max() < 1e-14
    assert np.abs(E[3:, 3:] - og.expm_taylor(S2)).max() < 1e-14
    assert np.abs(E[:3, 3:]).max() == 0.0


@pytest.mark.parametrize("g,sigma", [(8, 0.1), (16, 0.1), (32, 0.1), (64, 0.05), (128, 0.05), (16, 3.0)])
def test_gauge_orthogonal_and_matches_library(g, sigma):
    A = np.random.default_rng(g).normal(0, sigma, (g, g))
    G = og.gauge_from_A(A)
    assert np.abs(G.T @ G - np.eye(g)).max() < 1e-12
    assert abs(np.linalg.det(G) - 1.0) < 1e-10
    S = og.skew(A)
    assert np.abs(og.expm_taylor(S) @ og.expm_taylor(-S) - np.eye(g)).max() < 1e-12
    assert np.abs(G - scipy.linalg.expm(S)).max() < 1e-12
    assert np.abs(G - og.expm_pade13(S)).max() < 1e-12


def _cache(L=1, B=1, H=2, T=32, d=32, seed=0):
    return fl_bf16(np.random.default_rng(seed).standard_normal((L, 2, B, H, T, d)) * 3)


def test_apply_gauge_hand_example():
    # 2x2 rotation by th on group 0, identity on group 1 of a d=4 head.
    th = 0.5
    G = np.zeros((1, 2, 1, 2, 2, 2))
    G[..., 0, :, :] = [[np.cos(th), np.sin(th)], [-np.sin(th), np.cos(th)]]
    G[..., 1, :, :] = np.eye(2)
    x = np.zeros((1, 2, 1, 1, 1, 4))
    x[..., :] = [1.0, 0.0, 5.0, -2.0]
    y = og.apply_gauge(x, G)
    assert np.allclose(y[0, 0, 0, 0, 0], [np.cos(th), -np.sin(th), 5.0, -2.0], atol=1e-15)


def test_gauge_mixes_only_within_a_group():
    x = _cache()
    A = np.random.default_rng(1).normal(0, 0.3, (1, 2, 2, 4, 8, 8))
    G = og.gauge_from_A(A)
    y = og.apply_gauge(x, G)
    x2 = x.copy()
    x2[0, 1, 0, 1, 5, 8:16] += 1.0          # perturb group r=1 of one token
    y2 = og.apply_gauge(x2, G)
    diff = np.argwhere(y2 != y)
    assert len(diff) > 0
    assert set(map(tuple, diff[:, [0, 1, 2, 3, 4]])) == {(0, 1, 0, 1, 5)}
    assert diff[:, 5].min() >= 8 and diff[:, 5].max() < 16


def test_gauge_round_trip_and_energy():
    x = _cache()
    G = og.gauge_from_A(np.random.default_rng(2).normal(0, 0.2, (1, 2, 2, 2, 16, 16)))
    y = og.apply_gauge(x, G)
    assert abs((y ** 2).sum() / (x ** 2).sum() - 1) < 1e-13            # orthogonal: energy kept
    xr = og.apply_inverse_gauge(y, G)
    assert np.sqrt(((xr - x) ** 2).sum() / (x ** 2).sum()) < 1e-14     # G^T G x = x
    I = np.broadcast_to(np.eye(16), G.shape)
    assert np.array_equal(og.apply_gauge(x, I), x)


def test_f32_chain_against_exact_sequential_rationals():
    rng = np.random.default_rng(3)
    x = _cache(T=4, d=16)
    G32 = fl32(rng.normal(0, 0.3, (1, 2, 2, 1, 16, 16)))
    y = og.apply_gauge_f32_chain(x, G32)
    for (l, s, b, h, t) in [(0, 0, 0, 0, 0), (0, 1, 0, 1, 3), (0, 0, 0, 1, 2)]:
        for i in range(16):
            acc = 0.0
            for j in range(16):
                acc = _round_f32_exact(Fraction(G32[l, s, h, 0, i, j]) * Fraction(x[l, s, b, h, t, j]) + Fraction(acc))
            assert y[l, s, b, h, t, i] == acc


def test_f32_chain_within_fp32_dot_product_bound():
    x = _cache(T=64, d=32)
    G32 = fl32(og.gauge_from_A(np.random.default_rng(4).normal(0, 0.1, (1, 2, 2, 2, 16, 16))))
    y32 = og.apply_gauge_f32_chain(x, G32)
    y = og.apply_gauge(x, G32)
    # |fl(dot) - dot| <= gamma_g sum |G||x|, gamma_g = g u / (1 - g u), u = 2^-24
    absdot = og.apply_gauge(np.abs(x), np.abs(G32))
    u = 2.0 ** -24
    assert np.all(np.abs(y32 - y) <= 16 * u / (1 - 16 * u) * absdot)
    assert np.abs(y32 - y).max() > 0  # the chain really rounds
