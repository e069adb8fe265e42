"""Pins of the oracle's prefill attention (window and lookahead rows of the
target prefill, "Draft-based Approximate Inference for LLMs", section 关键设计,
SpecKV) against things other than itself: SciPy softmax / logsumexp over the
literal causal attention matrix, and closed forms (one key, identical keys,
two keys, a dominant key).  The input-key log-sum-exp it returns is also the
normaliser of the SpecKV scores, which ties it to the already-pinned scores."""
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


def _case(rng, g, nw, nl, n_in, d):
    q = _bits(rng.standard_normal((g, nw + nl, d)) / math.sqrt(d))
    k = _bits(rng.standard_normal((n_in + nl, d)))
    v = _bits(rng.standard_normal((n_in + nl, d)))
    return q, k, v


@pytest.mark.parametrize("g,nw,nl,n_in,d", [(1, 4, 4, 37, 8), (2, 16, 16, 120, 16), (3, 0, 5, 50, 8),
                                            (2, 7, 0, 64, 8), (1, 30, 3, 30, 4)])
def test_prefill_matches_bruteforce_attention(g, nw, nl, n_in, d):
    # the literal causal attention matrix over input + lookahead keys, its
    # softmax rows times V; the input-key normaliser by logsumexp
    rng = np.random.default_rng(g * 100 + n_in)
    q, k, v = _case(rng, g, nw, nl, n_in, d)
    out, lse = oracle.prefill_unit(q, k, v, nw, nl, n_in, scale=0.7)
    Q, K, V = _vals(q), _vals(k), _vals(v)
    R = nw + nl
    for h in range(g):
        for i in range(R):
            pos = n_in - nw + i if i < nw else n_in + i - nw
            z = 0.7 * K[:pos + 1] @ Q[h, i]
            np.testing.assert_allclose(out[h, i], softmax(z) @ V[:pos + 1], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(lse[h * R + i], logsumexp(z[:min(pos + 1, n_in)]), rtol=1e-13)


def test_prefill_sampled_rows_match_bruteforce():
    # the row-sampling form (used at full sizes) evaluates exactly the asked
    # rows, in the asked order, each equal to the literal attention row
    g, nw, nl, n_in, d = 3, 9, 6, 80, 8
    rng = np.random.default_rng(31)
    q, k, v = _case(rng, g, nw, nl, n_in, d)
    rows = [(2, 14), (0, 0), (1, 8), (1, 9), (2, 0), (0, 14)]
    out, lse = oracle.prefill_unit(q, k, v, nw, nl, n_in, scale=0.9, rows=rows)
    assert out.shape == (len(rows), d) and lse.shape == (len(rows),)
    Q, K, V = _vals(q), _vals(k), _vals(v)
    for j, (h, i) in enumerate(rows):
        pos = n_in - nw + i if i < nw else n_in + i - nw
        z = 0.9 * K[:pos + 1] @ Q[h, i]
        np.testing.assert_allclose(out[j], softmax(z) @ V[:pos + 1], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[j], logsumexp(z[:min(pos + 1, n_in)]), rtol=1e-13)


def test_prefill_closed_forms():
    d = 8
    rng = np.random.default_rng(5)
    # one visible key (a window row at position 0): out = v_0, lse = z_0
    q = _bits(rng.standard_normal((1, 1, d)))
    k = _bits(rng.standard_normal((1, d)))
    v = _bits(rng.standard_normal((1, d)))
    out, lse = oracle.prefill_unit(q, k, v, 1, 0, 1)
    np.testing.assert_array_equal(out[0, 0], _vals(v)[0])
    assert lse[0] == pytest.approx(float(_vals(q)[0, 0] @ _vals(k)[0]), rel=1e-15)
    # identical keys: uniform weights -> the mean of the visible values, lse = z + log c
    n_in, nl = 12, 3
    krow = rng.standard_normal(d)
    k = _bits(np.tile(krow, (n_in + nl, 1)))
    v = _bits(rng.standard_normal((n_in + nl, d)))
    q = _bits(rng.standard_normal((1, 2 + nl, d)))
    out, lse = oracle.prefill_unit(q, k, v, 2, nl, n_in)
    V = _vals(v)
    for i, c in enumerate([n_in - 1, n_in, n_in + 1, n_in + 2, n_in + 3]):
        np.testing.assert_allclose(out[0, i], V[:c].mean(axis=0), rtol=1e-13, atol=1e-15)
        z = float(_vals(q)[0, i] @ _vals(k)[0])
        assert lse[i] == pytest.approx(z + math.log(min(c, n_in)), rel=1e-13)
    # two keys: logistic weights sigma(z0 - z1), sigma(z1 - z0)
    k = _bits(rng.standard_normal((2, d)))
    v = _bits(rng.standard_normal((2, d)))
    q = _bits(rng.standard_normal((1, 1, d)))
    out, _ = oracle.prefill_unit(q, k, v, 1, 0, 2)
    z0, z1 = _vals(k) @ _vals(q)[0, 0]
    s = 1.0 / (1.0 + math.exp(z1 - z0))
    np.testing.assert_allclose(out[0, 0], s * _vals(v)[0] + (1 - s) * _vals(v)[1], rtol=1e-13)


def test_prefill_dominant_key_and_causality():
    # a huge logit on one key pulls every row that sees it onto its value;
    # rows before it never see it (causal)
    d, n_in, nw, nl = 8, 40, 6, 2
    rng = np.random.default_rng(9)
    qv = rng.standard_normal(d)
    qv /= np.linalg.norm(qv)
    q = _bits(np.tile(qv, (1, nw + nl, 1)))
    k = rng.standard_normal((n_in + nl, d)) * 0.01
    k[n_in - 3] = 80.0 * qv
    k = _bits(k)
    v = _bits(rng.standard_normal((n_in + nl, d)))
    out, lse = oracle.prefill_unit(q, k, v, nw, nl, n_in)
    V = _vals(v)
    for i in range(nw + nl):
        pos = n_in - nw + i if i < nw else n_in + i - nw
        if pos >= n_in - 3:
            np.testing.assert_allclose(out[0, i], V[n_in - 3], atol=1e-12)
        else:
            assert np.abs(out[0, i] - V[n_in - 3]).max() > 0.1


def test_prefill_lse_is_the_scores_normaliser():
    # lse_in of every row is the log-normaliser under which that row's softmax
    # over the input keys sums to one: exp(z - lse_in) summed over the
    # prefix and window keys, over all rows, equals the (pinned) SpecKV
    # scores plus window mass, which sum to g * R
    rng = np.random.default_rng(13)
    g, nw, nl, n_in, d = 2, 5, 4, 33, 8
    q, k, v = _case(rng, g, nw, nl, n_in, d)
    _, lse = oracle.prefill_unit(q, k, v, nw, nl, n_in)
    s, wm = oracle.speckv_unit(q, k[:n_in], nw, nl)
    Q, K = _vals(q), _vals(k)
    acc = np.zeros(n_in)
    R = nw + nl
    for h in range(g):
        for i in range(R):
            pos = n_in - nw + i if i < nw else n_in + i - nw
            c = min(pos + 1, n_in)
            acc[:c] += np.exp(K[:c] @ Q[h, i] - lse[h * R + i])
    np.testing.assert_allclose(acc, np.concatenate([s, wm]), rtol=1e-12, atol=1e-15)
    assert acc.sum() == pytest.approx(g * R, rel=1e-12)
