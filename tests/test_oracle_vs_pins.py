"""Pins of the oracle's Vertical-Slash sparse attention against things other
than itself: SciPy softmax over the literal masked attention matrix, dense
causal attention when the pattern covers every key, and closed forms (a
token alone with itself; one extra key: logistic weights)."""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
import workloads as W


def _bits(x):
    return W.bf16_bits(np.asarray(x, np.float32))


def _vals(b):
    return W.bf16_decode(b).astype(np.float64)


def _case(rng, g, n_q, n, d):
    q = _bits(rng.standard_normal((g, n_q, d)) / math.sqrt(d))
    k = _bits(rng.standard_normal((n, d)))
    v = _bits(rng.standard_normal((n, d)))
    return q, k, v


def _bruteforce(q, k, v, vertical, slash, scale):
    Q, K, V = _vals(q), _vals(k), _vals(v)
    g, n_q, _ = Q.shape
    n = K.shape[0]
    vs, ss = set(int(x) for x in vertical), set(int(x) for x in slash)
    out = np.zeros(Q.shape)
    lse = np.zeros(g * n_q)
    for h in range(g):
        for i in range(n_q):
            p = n - n_q + i
            mask = np.array([j <= p and (j == p or j in vs or (p - j) in ss) for j in range(n)])
            z = np.where(mask, scale * (K @ Q[h, i]), -np.inf)
            out[h, i] = softmax(z) @ V
            lse[h * n_q + i] = logsumexp(z)
    return out, lse


@pytest.mark.parametrize("g,n_q,n,d,nv,ns", [(1, 10, 40, 8, 5, 3), (2, 33, 33, 16, 7, 6), (3, 5, 90, 8, 20, 1),
                                             (1, 64, 200, 4, 0, 9), (2, 20, 60, 8, 11, 0)])
def test_vs_matches_masked_bruteforce(g, n_q, n, d, nv, ns):
    rng = np.random.default_rng(n * 10 + nv)
    q, k, v = _case(rng, g, n_q, n, d)
    vert = np.sort(rng.choice(n, size=nv, replace=False))
    sl = np.sort(rng.choice(n, size=ns, replace=False))
    out, lse = oracle.vs_attention_unit(q, k, v, vert, sl, scale=0.9)
    ref, rlse = _bruteforce(q, k, v, vert, sl, 0.9)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, rlse, rtol=1e-13)


def test_vs_sampled_rows_match_bruteforce():
    # the row-sampling form (used at full sizes) evaluates exactly the asked
    # rows, in the asked order
    g, n_q, n, d = 2, 30, 70, 8
    rng = np.random.default_rng(77)
    q, k, v = _case(rng, g, n_q, n, d)
    vert = np.sort(rng.choice(n, size=9, replace=False))
    sl = np.sort(rng.choice(n, size=5, replace=False))
    rows = [(1, 29), (0, 0), (1, 3), (0, 17)]
    out, lse = oracle.vs_attention_unit(q, k, v, vert, sl, scale=0.8, rows=rows)
    ref, rlse = _bruteforce(q, k, v, vert, sl, 0.8)
    for j, (h, i) in enumerate(rows):
        np.testing.assert_allclose(out[j], ref[h, i], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[j], rlse[h * n_q + i], rtol=1e-13)


def test_vs_full_pattern_is_dense_causal_attention():
    # every key vertical, or every offset a slash: plain causal attention,
    # which is the oracle's (pinned) prefill attention with no lookahead
    rng = np.random.default_rng(3)
    g, n_q, n, d = 2, 12, 50, 8
    q, k, v = _case(rng, g, n_q, n, d)
    dense, dlse = oracle.prefill_unit(q, k, v, n_q, 0, n)
    for vert, sl in ((np.arange(n), []), ([], np.arange(n))):
        out, lse = oracle.vs_attention_unit(q, k, v, vert, sl)
        np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, dlse, rtol=1e-13)


def test_vs_closed_forms():
    rng = np.random.default_rng(4)
    g, n_q, n, d = 1, 6, 20, 8
    q, k, v = _case(rng, g, n_q, n, d)
    Q, K, V = _vals(q), _vals(k), _vals(v)
    # empty pattern: each token sees only itself
    out, lse = oracle.vs_attention_unit(q, k, v, [], [])
    for i in range(n_q):
        p = n - n_q + i
        np.testing.assert_array_equal(out[0, i], V[p])
        assert lse[i] == pytest.approx(float(Q[0, i] @ K[p]), rel=1e-14)
    # slash {1}: itself and its predecessor; vertical {0}: itself and key 0
    for vert, sl, other in (([], [1], lambda p: p - 1), ([0], [], lambda p: 0)):
        out, _ = oracle.vs_attention_unit(q, k, v, vert, sl)
        for i in range(n_q):
            p = n - n_q + i
            a, b = float(Q[0, i] @ K[p]), float(Q[0, i] @ K[other(p)])
            w = 1.0 / (1.0 + math.exp(b - a))
            np.testing.assert_allclose(out[0, i], w * V[p] + (1 - w) * V[other(p)], rtol=1e-12, atol=1e-15)
