"""Plant plausible mistakes in the oracle (CPU only) and check that a pin
catches each one: a transposed gauge, a dropped DCT normalization, a wrong
radius denominator, a sign flip in the gradient, a dropped FMA midpoint fix,
a swapped packing bit order and truncating instead of RNE rounding."""
import numpy as np
import pytest

import oracle.fpround as fpr
import oracle.gauge as og
import oracle.quant as oq
import oracle.spectral as sp
from tests import test_oracle_fpround as t_fp
from tests import test_oracle_gauge as t_g
from tests import test_oracle_quant as t_q
from tests import test_oracle_spectral as t_sp


def _fails(fn, *a):
    with pytest.raises(AssertionError):
        fn(*a)


def test_transposed_gauge_is_caught(monkeypatch):
    orig = og.apply_gauge
    monkeypatch.setattr(og, "apply_gauge", lambda kv, G: orig(kv, np.swapaxes(np.asarray(G), -1, -2)))
    _fails(t_g.test_apply_gauge_hand_example)


def test_unnormalized_dct_is_caught(monkeypatch):
    orig = sp.dct_matrix

    def bad(N):
        C = orig(N)
        C[0, :] = np.sqrt(2.0 / N)   # alpha_0 = sqrt(2/N) by mistake
        return C
    monkeypatch.setattr(sp, "dct_matrix", bad)
    _fails(t_sp.test_dct_orthonormal, 16)


def test_radius_denominator_is_caught(monkeypatch):
    def bad(tb, d):
        u = np.arange(tb, dtype=np.float64)[:, None] / tb
        v = np.arange(d, dtype=np.float64)[None, :] / d
        return np.sqrt(u * u + v * v) / np.sqrt(2.0)
    monkeypatch.setattr(sp, "radius", bad)
    _fails(t_sp.test_radius_corners)


def test_gradient_sign_is_caught(monkeypatch):
    orig = sp.grad_U
    monkeypatch.setattr(sp, "grad_U", lambda *a, **k: -orig(*a, **k))
    _fails(t_sp.test_grad_G_finite_differences)


def test_dropped_rate_term_is_caught(monkeypatch):
    orig = sp.grad_U
    monkeypatch.setattr(sp, "grad_U", lambda U, lf, E, n, tau=sp.TAU, lambda_f=1.0, lambda_r=0.02:
                        orig(U, lf, E, n, tau, lambda_f, 0.0))
    _fails(t_sp.test_grad_G_finite_differences)


def test_naive_fma_is_caught(monkeypatch):
    monkeypatch.setattr(fpr, "fma_f32", lambda a, b, c: fpr.fl32(np.asarray(a, np.float64) * b + c))
    monkeypatch.setattr(t_fp, "fma_f32", fpr.fma_f32)
    _fails(t_fp.test_fma_f32_double_rounding_traps)


def test_big_endian_packing_is_caught(monkeypatch):
    orig = oq.pack_codes

    def bad(q, bits):   # MSB-first bit order inside each byte
        return np.packbits(np.unpackbits(orig(q, bits), axis=-1, bitorder="little"), axis=-1, bitorder="big")
    monkeypatch.setattr(oq, "pack_codes", bad)
    _fails(t_q.test_packing_golden, 4, [1, 2, 3, 4], bytes.fromhex("2143"))


def test_truncating_quantizer_is_caught(monkeypatch):
    def bad(y, z, s, bits):
        qmax = 2 ** bits - 1
        y = np.asarray(y, np.float64)
        z = np.broadcast_to(np.asarray(z, np.float64), y.shape)
        s = np.broadcast_to(np.asarray(s, np.float64), y.shape)
        nz = s != 0
        t = fpr.fl32(fpr.fl32(y - z) * fpr.fl32(1.0 / np.where(nz, s, 1.0)))
        return np.where(nz, np.clip(np.floor(t), 0, qmax), 0).astype(np.int64)
    monkeypatch.setattr(oq, "quantize", bad)
    _fails(t_q.test_rne_ties_go_to_even)
