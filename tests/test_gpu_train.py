"""GPU parity of the gauge-training step against the oracle: dL/dA through the
exp Frechet adjoint (cg_gauge_grad, fp64 inside, fp32 out) within 1e-6 of the
largest entry; AdamW (cg_adamw_step, fp32) within 1e-6 relative after several
steps; a whole training step on a small cache; and a short training run whose
objective decreases."""
import numpy as np
import pytest
import torch

from oracle import gauge as og
from oracle import spectral as sp
from oracle import train as otr
from quantization_cg_encode_b200 import cg, synth
from quantization_cg_encode_b200.train import GaugeTrainer
from tests.gpu_util import bf16_np, need_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("g", [6, 8, 16, 20, 32])
def test_gauge_grad_matches_frechet_adjoint(g):
    need_gpu()
    rng = np.random.default_rng(g)
    n = 37
    A = (0.1 * rng.standard_normal((n, g, g))).astype(np.float32)
    dG = (rng.standard_normal((n, g, g)) * 10.0 ** rng.uniform(-6, 2, (n, 1, 1))).astype(np.float32)
    A[0] = 0.0                       # S = 0: dA = dG - dG^T
    A[1] *= 40.0                     # a large skew part: several squarings
    dG[2] = 0.0                      # zero gradient
    dA = torch.empty((n, g, g), dtype=torch.float32, device="cuda")
    cg.cg_gauge_grad(torch.from_numpy(A).cuda(), torch.from_numpy(dG).cuda(), dA)
    cg.cg_sync_status()
    got = dA.cpu().numpy().astype(np.float64)
    ref = sp.grad_A(A.astype(np.float64), dG.astype(np.float64))
    for i in range(n):
        scale = np.abs(ref[i]).max()
        assert np.abs(got[i] - ref[i]).max() <= 1e-6 * max(scale, 1e-30), i
    assert np.allclose(got, -np.swapaxes(got, -1, -2))          # dA is antisymmetric
    assert np.allclose(got[0], dG[0] - dG[0].T, rtol=1e-6, atol=1e-6 * np.abs(dG[0]).max())
    assert not got[2].any()


def test_adamw_matches_oracle():
    need_gpu()
    rng = np.random.default_rng(3)
    n = 10_000
    p = rng.standard_normal(n).astype(np.float32)
    hp = dict(lr=2e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    P, M, V = (torch.from_numpy(p.copy()).cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda"))
    rp, rm, rv = p.astype(np.float64), np.zeros(n), np.zeros(n)
    sum_g, sum_g2 = np.zeros(n), np.zeros(n)  # magnitudes the fp32 moments are accumulated from
    for t in range(1, 6):
        gr = (rng.standard_normal(n) * 10.0 ** rng.uniform(-4, 1, n)).astype(np.float32)
        cg.cg_adamw_step(P, torch.from_numpy(gr).cuda(), M, V, cg.adamw_desc(**hp), t)
        rp, rm, rv = otr.adamw_step(rp, gr.astype(np.float64), rm, rv, t, **hp)
        sum_g += np.abs(gr)
        sum_g2 += gr.astype(np.float64) ** 2
    cg.cg_sync_status()
    assert np.allclose(P.cpu().numpy(), rp, rtol=1e-6, atol=1e-7)
    # each moment is a sum of terms of opposite signs: its fp32 error scales with the terms
    assert np.all(np.abs(M.cpu().numpy() - rm) <= 1e-6 * sum_g)
    assert np.all(np.abs(V.cpu().numpy() - rv) <= 1e-6 * sum_g2)


def test_training_step_matches_oracle():
    """One window of 1 x 2 x 1 x 2 x 256 x 128, g = 16: G, the window's totals and
    the updated A against the oracle's step.  Adam's first step moves each entry by
    about lr sign(dA); entries whose oracle gradient is within the device's dG
    accuracy of zero (|dA| < 1e-3 max |dA|) may take the other sign."""
    need_gpu()
    L, B, H, T, d = 1, 1, 2, 256, 128
    kv = synth.kv_cache(L, B, H, T, d, seed=4, device="cuda", n_outliers=2)
    A0 = synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=4)
    tr = GaugeTrainer(A0.clone().cuda(), kv.shape)
    tot = tr.step(kv).cpu().numpy()
    A1 = tr.A.cpu().numpy().astype(np.float64)
    rA, _, _, rtot = otr.train_step(A0.numpy().astype(np.float64), bf16_np(kv), np.zeros(A0.shape),
                                    np.zeros(A0.shape), 1)
    assert np.all(np.abs(tot - rtot) <= 1e-4 * np.abs(rtot))
    dA_ref = sp.grad_A(A0.numpy().astype(np.float64),
                       sp.spectral_stats(bf16_np(kv), og.gauge_from_A(A0.numpy().astype(np.float64)),
                                         want_grad=True)["dG"])
    sure = np.abs(dA_ref) >= 1e-3 * np.abs(dA_ref).max()
    assert np.all(np.abs(A1 - rA)[sure] <= 1e-6 + 1e-5 * np.abs(rA)[sure])
    assert np.all(np.abs(A1 - rA)[~sure] <= 2.2e-3)


def test_short_training_run_reduces_the_objective():
    """Four windows of a small cache, six epochs: the objective and the frequency
    term fall, and the spectral concentration 1 - L_freq rises."""
    need_gpu()
    L, B, H, T, d = 1, 1, 2, 512, 128
    windows = [synth.kv_cache(L, B, H, T, d, seed=40 + w, device="cuda", n_outliers=2) for w in range(4)]
    A = synth.gauge_params(L, H, 8, 16, sigma=0.1, seed=5).cuda()
    tr = GaugeTrainer(A, windows[0].shape, hp=cg.adamw_desc(lr=1e-2))
    hist = [tr.epoch(windows) for _ in range(6)]
    cg.cg_sync_status()
    (L0, F0), (L5, F5) = hist[0], hist[-1]
    assert L5 < L0 and F5 < F0, hist
    assert np.isfinite(np.array(hist)).all()
