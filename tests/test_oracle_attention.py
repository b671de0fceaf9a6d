"""Pins of the oracle's decode-step attention: one token returns its value, a
zero query averages the values, a brute-force loop over heads and tokens, and
the grouped-query head mapping."""
import numpy as np

from oracle import attention as oa


def test_single_token_returns_its_value():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((2, 4, 8)), rng.standard_normal((2, 2, 1, 8)), rng.standard_normal((2, 2, 1, 8))
    out = oa.softmax_attention(q, k, v, 0.3)
    assert np.allclose(out, np.repeat(v[:, :, 0], 2, axis=1), rtol=1e-15)


def test_zero_query_averages_values():
    rng = np.random.default_rng(1)
    k, v = rng.standard_normal((3, 5, 8)), rng.standard_normal((3, 5, 8))
    out = oa.softmax_attention(np.zeros((3, 8)), k, v, 1.0)
    assert np.allclose(out, v.mean(axis=1), rtol=1e-14)


def test_brute_force_and_head_mapping():
    rng = np.random.default_rng(2)
    Hq, H, n, d = 6, 2, 7, 5
    q, k, v = rng.standard_normal((Hq, d)), rng.standard_normal((H, n, d)), rng.standard_normal((H, n, d))
    out = oa.softmax_attention(q, k, v, 0.7)
    for j in range(Hq):
        h = j // (Hq // H)  # query heads 0-2 use KV head 0, 3-5 use KV head 1
        s = [0.7 * sum(q[j, c] * k[h, t, c] for c in range(d)) for t in range(n)]
        e = [np.exp(x - max(s)) for x in s]
        ref = [sum(e[t] * v[h, t, c] for t in range(n)) / sum(e) for c in range(d)]
        assert np.allclose(out[j], ref, rtol=1e-13)
