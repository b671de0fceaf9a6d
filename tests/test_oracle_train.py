"""Pins of the oracle's AdamW and control gauges: torch's AdamW (a library
routine) on the same trajectory, the first step's closed form, brute-force Gram
sums, the Hadamard matrix's defining properties and the KLT's diagonalization."""
import numpy as np
import pytest
import torch

from oracle import controls as oc
from oracle import train as ot


def test_adamw_matches_torch_over_several_steps():
    rng = np.random.default_rng(0)
    p0 = rng.standard_normal(50)
    grads = rng.standard_normal((6, 50)) * np.array([1e-3, 1.0, 10.0, 0.1, 5.0, 1e-2])[:, None]
    hp = dict(lr=3e-3, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.05)
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"])
    p, m, v = p0.copy(), np.zeros(50), np.zeros(50)
    for t, gr in enumerate(grads, 1):
        p, m, v = ot.adamw_step(p, gr, m, v, t, **hp)
        tp.grad = torch.tensor(gr, dtype=torch.float64)
        opt.step()
        assert np.allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-14)


def test_adamw_first_step_closed_form():
    """Step 1: m_hat = g, v_hat = g^2, so p -= lr (g / (|g| + eps) + wd p)."""
    p, g = np.array([1.0, -2.0, 0.5, 0.0]), np.array([0.3, -1e-3, 0.0, 2.0])
    out, m, v = ot.adamw_step(p, g, np.zeros(4), np.zeros(4), 1, lr=0.1, eps=1e-8, weight_decay=0.01)
    assert np.allclose(out, p - 0.1 * (g / (np.abs(g) + 1e-8) + 0.01 * p), rtol=1e-14, atol=1e-16)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def test_gram_brute_force():
    rng = np.random.default_rng(1)
    kv = rng.standard_normal((1, 2, 2, 2, 8, 32))
    C = oc.gram(kv, 16, t0=2, nt=5)
    ref = np.zeros((1, 2, 2, 2, 16, 16))
    for s in range(2):
        for h in range(2):
            for r in range(2):
                for b in range(2):
                    for t in range(2, 7):
                        x = kv[0, s, b, h, t, 16 * r:16 * r + 16]
                        ref[0, s, h, r] += np.outer(x, x)
    assert np.allclose(C, ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("g", [2, 8, 16, 32, 128])
def test_hadamard_properties(g):
    H = oc.hadamard(g)
    assert np.allclose(np.abs(H), 1.0 / np.sqrt(g))
    assert np.allclose(H @ H.T, np.eye(g), atol=1e-14) and np.allclose(H, H.T)
    assert np.all(H[0] > 0) and np.all(H[:, 0] > 0)


def test_klt_diagonalizes_second_moments():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((500, 16)) @ rng.standard_normal((16, 16))
    C = X.T @ X
    G, w = oc.klt(C)
    D = G @ C @ G.T
    assert np.allclose(G @ G.T, np.eye(16), atol=1e-12)
    assert np.allclose(D, np.diag(np.diag(D)), atol=1e-9 * np.abs(D).max())
    assert np.allclose(np.diag(D), w, rtol=1e-10) and np.all(np.diff(w) <= 0)
    assert np.all(G[np.arange(16), np.argmax(np.abs(G), 1)] > 0)
