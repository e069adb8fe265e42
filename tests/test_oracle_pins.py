"""Pins of the fp64 oracle against things other than itself.

Each test names what fixes the expected value: a library routine applied to
the literal definition (brute force), a hand-worked closed form, an
invariant of softmax attention, or Theorem 1 of "Draft-based Approximate
Inference for LLMs" (section 关键设计, SpecKV).  Together they are chosen so
that a dropped term, a wrong sign, an off-by-one position, a transposed
operand or a wrong tie rule in the oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as W
from tests import bruteforce as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "speckv_handworked.json")


def _rand_case(rng, g, n_window, n_lookahead, n_in, d, bf16=False):
    q = rng.standard_normal((g, n_window + n_lookahead, d)) / math.sqrt(d)
    k = rng.standard_normal((n_in, d))
    if bf16:
        return W.bf16_bits(q.astype(np.float32)), W.bf16_bits(k.astype(np.float32))
    return q, k


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("g,n_window,n_lookahead,n_in,d", [
    (1, 4, 4, 37, 8), (2, 16, 16, 120, 16), (3, 0, 5, 50, 8), (2, 7, 0, 64, 8),
    (4, 1, 3, 9, 4), (1, 30, 2, 30, 8),   # window covers every input key
])
def test_speckv_matches_bruteforce(g, n_window, n_lookahead, n_in, d):
    rng = np.random.default_rng(g * 1000 + n_in)
    q, k = _rand_case(rng, g, n_window, n_lookahead, n_in, d)
    s, wm = oracle.speckv_unit(q, k, n_window, n_lookahead)
    bs, bwm = bf.speckv_unit(q, k, n_window, n_lookahead)
    np.testing.assert_allclose(s, bs, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(wm, bwm, rtol=1e-12, atol=1e-15)


def test_speckv_bf16_entry_matches_decoded_f64():
    rng = np.random.default_rng(7)
    qb, kb = _rand_case(rng, 2, 8, 8, 100, 16, bf16=True)
    s1, w1 = oracle.speckv_unit(qb, kb, 8, 8)
    s2, w2 = oracle.speckv_unit(W.bf16_decode(qb).astype(np.float64),
                                W.bf16_decode(kb).astype(np.float64), 8, 8)
    assert np.array_equal(s1, s2) and np.array_equal(w1, w2)


def test_speckv_scale_argument():
    rng = np.random.default_rng(3)
    q, k = _rand_case(rng, 2, 3, 4, 40, 8)
    s1, _ = oracle.speckv_unit(q, k, 3, 4, scale=0.37)
    s2, _ = bf.speckv_unit(q, k, 3, 4, scale=0.37)
    np.testing.assert_allclose(s1, s2, rtol=1e-12)


def test_speckv_lse_is_row_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(11)
    q, k = _rand_case(rng, 2, 5, 3, 33, 8)
    _, _, lse = oracle.speckv_unit(q, k, 5, 3, with_lse=True)
    n_in = 33
    for h in range(2):
        for i in range(8):
            pos = n_in - 5 + i if i < 5 else n_in + i - 5
            c = min(pos, n_in - 1) + 1
            np.testing.assert_allclose(lse[h * 8 + i], logsumexp(q[h, i] @ k[:c].T), rtol=1e-13)


# ---------------------------------------------------------------- hand-worked
def _frac(s):
    return float(Fraction(s))


def _logit(s):
    s = s.strip()
    return 0.0 if s == "0" else math.log(float(s.split()[1]))


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_handworked_cases(case):
    n_in, nw, nl = case["n_in"], case["n_window"], case["n_lookahead"]
    z = [_logit(s) for s in case["logits"]]
    q = np.zeros((1, nw + nl, 2))
    q[:, :, 0] = 1.0
    k = np.zeros((n_in, 2))
    k[:, 0] = z
    s, wm = oracle.speckv_unit(q, k, nw, nl)
    np.testing.assert_allclose(s, [_frac(x) for x in case["scores"]], rtol=1e-14)
    np.testing.assert_allclose(wm, [_frac(x) for x in case["window_mass"]], rtol=1e-14)
    for key in ("topk", "topk_pool3"):
        if key in case:
            t = case[key]
            idx = oracle.topk_with_tail(oracle.maxpool(s, t["pool"]), t["c_max"], nw)
            assert idx.tolist() == t["idx"]


def test_one_dominant_key_closed_form():
    # logit L on key jd, 0 elsewhere: p_dom = e^L/(e^L+c-1), others 1/(e^L+c-1)
    g, nw, nl, n_in, Lg, jd = 3, 6, 5, 40, 2.5, 17
    q = np.zeros((g, nw + nl, 4)); q[..., 1] = 1.0
    k = np.zeros((n_in, 4)); k[jd, 1] = Lg
    s, wm = oracle.speckv_unit(q, k, nw, nl)
    n_pre = n_in - nw
    cs = [n_pre + i + 1 for i in range(nw)] + [n_in] * nl
    e = math.exp(Lg)
    exp_other = np.zeros(n_in)
    dom = 0.0
    for c in cs:
        exp_other[:c] += 1.0 / (e + c - 1)
        dom += e / (e + c - 1)
    exp_other[jd] = dom
    exp_other *= g
    np.testing.assert_allclose(s, exp_other[:n_pre], rtol=1e-13)
    np.testing.assert_allclose(wm, exp_other[n_pre:], rtol=1e-13)
    assert int(np.argmax(s)) == jd


def test_uniform_keys_closed_form_and_ties():
    # identical keys: every visible key gets 1/c from each row
    g, nw, nl, n_in, d = 2, 16, 16, 512, 8
    rng = np.random.default_rng(5)
    q = rng.standard_normal((g, nw + nl, d))
    k = np.tile(rng.standard_normal((1, d)), (n_in, 1))
    s, wm = oracle.speckv_unit(q, k, nw, nl)
    n_pre = n_in - nw
    expect = g * (nl / n_in + sum(1.0 / (n_pre + i + 1) for i in range(nw)))
    np.testing.assert_allclose(s, expect, rtol=1e-12)
    idx = oracle.topk_with_tail(oracle.maxpool(s, 7), 64, nw)
    # exact ties everywhere -> the lowest indices win
    assert idx.tolist() == list(range(64)) + list(range(n_pre, n_in))


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("seed", range(5))
def test_total_mass_equals_rows(seed):
    rng = np.random.default_rng(seed)
    g, nw, nl, n_in = 1 + seed % 3, 3 + seed, 2 * seed, 60 + 7 * seed
    q, k = _rand_case(rng, g, nw, nl, n_in, 16)
    s, wm = oracle.speckv_unit(q, k, nw, nl)
    assert abs(s.sum() + wm.sum() - g * (nw + nl)) < 1e-10
    assert (s >= 0).all() and (wm >= 0).all()


def test_window_rows_are_causal():
    # a huge logit on the last input key must not reach window rows before it
    nw, nl, n_in = 4, 0, 20
    q = np.zeros((1, nw, 2)); q[..., 0] = 1.0
    k = np.zeros((n_in, 2)); k[-1, 0] = 30.0
    s, wm = oracle.speckv_unit(q, k, nw, nl)
    # rows 0..2 see uniform logits over their visible keys; row 3 is dominated
    n_pre = n_in - nw
    expect = sum(1.0 / (n_pre + i + 1) for i in range(3)) + 1.0 / (math.exp(30) + n_in - 1)
    np.testing.assert_allclose(s, expect, rtol=1e-12)


def test_selection_invariants_random():
    rng = np.random.default_rng(9)
    for trial in range(30):
        n = int(rng.integers(1, 300))
        kk = int(rng.integers(0, 350))
        tail = int(rng.integers(0, 20))
        vals = rng.integers(0, 12, size=n).astype(np.float64)   # many exact ties
        idx = oracle.topk_with_tail(vals, kk, tail)
        ref = bf.topk_with_tail(vals, kk, tail)
        assert idx.tolist() == ref.tolist()
        c = min(kk, n)
        assert len(idx) == c + tail
        assert np.all(np.diff(idx[:c]) > 0)
        assert idx[c:].tolist() == list(range(n, n + tail))


# ---------------------------------------------------------------- pooling
def test_maxpool_matches_library_filter():
    rng = np.random.default_rng(1)
    for n in (1, 2, 3, 7, 8, 100, 1001):
        s = rng.random(n)
        for kernel in (1, 3, 7, 9):
            np.testing.assert_array_equal(oracle.maxpool(s, kernel), bf.maxpool(s, kernel))


def test_maxpool_plateau_by_hand():
    s = np.zeros(11); s[3] = 5.0
    assert oracle.maxpool(s, 7).tolist() == [5.0] * 7 + [0.0] * 4


@pytest.mark.parametrize("kernel", [1, 3, 7, 9, 31])
def test_avgpool_matches_library_filters(kernel):
    # the average over the window clipped to the row: a library box filter
    # with zero padding, divided by the same filter applied to ones
    rng = np.random.default_rng(kernel)
    for n in (1, 2, 5, 40, 333):
        s = rng.random(n)
        np.testing.assert_allclose(oracle.avgpool(s, kernel), bf.avgpool(s, kernel), rtol=1e-13, atol=0)


def test_avgpool_by_hand():
    # kernel 3 on (0, 3, 6, 9): ends average two values, the middle three
    assert oracle.avgpool(np.array([0.0, 3.0, 6.0, 9.0]), 3).tolist() == [1.5, 3.0, 6.0, 7.5]
    # a kernel wider than the row averages the whole row everywhere
    assert oracle.avgpool(np.array([1.0, 2.0, 6.0]), 9).tolist() == [3.0, 3.0, 3.0]
    assert oracle.pool(np.array([1.0, 5.0, 2.0]), 3, "avg").tolist() == [3.0, 8.0 / 3.0, 3.5]
    assert oracle.pool(np.array([1.0, 5.0, 2.0]), 3, "max").tolist() == [5.0, 5.0, 5.0]


def test_avgpool_rejects_even_kernel():
    with pytest.raises(ValueError):
        oracle.avgpool(np.zeros(5), 2)


def test_maxpool_rejects_even_kernel():
    with pytest.raises(ValueError):
        oracle.maxpool(np.zeros(5), 4)


# ---------------------------------------------------------------- compaction
def test_gather_matches_take_bitexact():
    rng = np.random.default_rng(2)
    src = rng.integers(0, 2 ** 16, size=(300, 64), dtype=np.uint16)
    idx = np.sort(rng.choice(300, size=77, replace=False)).astype(np.int32)
    np.testing.assert_array_equal(oracle.gather_rows(src, idx), np.take(src, idx, axis=0))


def test_gather_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.gather_rows(np.zeros((4, 2), np.uint16), np.array([4], np.int32))


# ---------------------------------------------------------------- SpecPC
def _specpc_case(rng, L, hq, hkv, n_in, n_lookahead, Wr, d):
    T = n_in + n_lookahead - 1
    q_all = rng.standard_normal((L, hq, T, d)) / math.sqrt(d)
    k = rng.standard_normal((L, hkv, n_in, d))
    return q_all, k


@pytest.mark.parametrize("L,l_skip,hq,hkv,n_in,n_lookahead,Wr", [
    (3, 1, 4, 2, 40, 1, 8), (2, 0, 3, 1, 25, 4, 6), (4, 3, 2, 2, 30, 1, 30), (1, 0, 1, 1, 10, 1, 1),
])
def test_specpc_matches_full_attention_tensor(L, l_skip, hq, hkv, n_in, n_lookahead, Wr):
    rng = np.random.default_rng(L * 100 + n_in)
    q_all, k = _specpc_case(rng, L, hq, hkv, n_in, n_lookahead, Wr, 8)
    w = W.specpc_row_weights(Wr)
    T = q_all.shape[2]
    got = oracle.specpc_batch(q_all[:, :, T - Wr:], k, w, l_skip, n_lookahead)
    ref = bf.specpc_batch(q_all, k, w, l_skip)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-16)


@pytest.mark.parametrize("L,l_skip,hq,hkv,n_in,n_lookahead,Wr,d", [
    (3, 1, 4, 2, 40, 1, 8, 8),     # every dimension distinct from the others
    (2, 0, 6, 3, 23, 3, 5, 16),
    (4, 2, 2, 1, 17, 1, 16, 4),    # W close to n_in
])
def test_specpc_bf16_entry_matches_bruteforce_on_decoded_values(L, l_skip, hq, hkv, n_in, n_lookahead, Wr, d):
    # The bf16 entry decodes q [L][Hq][W][d] and k [L][Hkv][n_in][d] itself;
    # it must equal the float entry on the decoded values exactly and the
    # brute-force draft attention tensor built from those values.  A size,
    # offset or tensor mix-up in the decode (say, q's element count used for
    # k) changes these numbers.
    rng = np.random.default_rng(L * 1000 + n_in * 10 + d)
    T = n_in + n_lookahead - 1
    q_all = W.bf16_bits((rng.standard_normal((L, hq, T, d)) / math.sqrt(d)).astype(np.float32))
    kb = W.bf16_bits(rng.standard_normal((L, hkv, n_in, d)).astype(np.float32))
    qb = np.ascontiguousarray(q_all[:, :, T - Wr:])
    w = W.specpc_row_weights(Wr)
    got = oracle.specpc_batch(qb, kb, w, l_skip, n_lookahead)
    f64 = oracle.specpc_batch(W.bf16_decode(qb).astype(np.float64), W.bf16_decode(kb).astype(np.float64),
                              w, l_skip, n_lookahead)
    assert np.array_equal(got, f64)
    ref = bf.specpc_batch(W.bf16_decode(q_all).astype(np.float64), W.bf16_decode(kb).astype(np.float64), w, l_skip)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-16)


def test_specpc_zero_weight_rows_contribute_nothing():
    # rows of weight 0 drop out of the weighted mean: the brute-force
    # attention tensor with the same weights, and, where only the zero-weight
    # (latest) rows see a key, a score of exactly 0
    rng = np.random.default_rng(31)
    L, hq, hkv, n_in, nl, Wr, d = 2, 4, 2, 30, 1, 6, 8
    T = n_in + nl - 1
    q_all = rng.standard_normal((L, hq, T, d)) / math.sqrt(d)
    k = rng.standard_normal((L, hkv, n_in, d))
    w = np.array([0.3, 0.0, 1.0, 0.5, 0.0, 0.0])
    got = oracle.specpc_batch(q_all[:, :, T - Wr:], k, w, 0, nl)
    np.testing.assert_allclose(got, bf.specpc_batch(q_all, k, w, 0), rtol=1e-12, atol=1e-16)
    # the last two rows (positions n_in-2, n_in-1) have weight 0 and are the
    # only rows that see keys n_in-2 and n_in-1; row 3 (weight 0.5) sees n_in-3
    assert got[n_in - 1] == 0.0 and got[n_in - 2] == 0.0 and got[n_in - 3] > 0.0


def test_specpc_single_row_is_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 1, 8)); k = rng.standard_normal((1, 1, 50, 8))
    got = oracle.specpc_batch(q, k, [1.0], 0, 1)
    np.testing.assert_allclose(got, softmax(q[0, 0, 0] @ k[0, 0].T), rtol=1e-13)


def test_specpc_uniform_weights_reduce_to_speckv_window():
    # one layer, one head, uniform weights, n_lookahead=1: rows are the last W
    # input tokens, i.e. SpecKV window rows; SpecPC = column sum / W
    rng = np.random.default_rng(6)
    Wr, n_in = 9, 45
    q = rng.standard_normal((1, 1, Wr, 8)); k = rng.standard_normal((1, 1, n_in, 8))
    got = oracle.specpc_batch(q, k, np.ones(Wr), 0, 1)
    s, wm = oracle.speckv_unit(q[0], k[0, 0], Wr, 0)
    np.testing.assert_allclose(got, np.concatenate([s, wm]) / Wr, rtol=1e-13)


def test_specpc_head_max_and_layer_mean():
    rng = np.random.default_rng(8)
    L, hq, hkv, n_in, Wr = 3, 4, 2, 30, 5
    q = rng.standard_normal((L, hq, Wr, 8)); k = rng.standard_normal((L, hkv, n_in, 8))
    w = W.specpc_row_weights(Wr)
    # identical query heads -> head max equals the single-head value
    q_same = np.repeat(q[:, :1], hq, axis=1)
    k_same = np.repeat(k[:, :1], hkv, axis=1)
    one = oracle.specpc_batch(q_same[:, :1], k_same[:, :1], w, 1, 1)
    allh = oracle.specpc_batch(q_same, k_same, w, 1, 1)
    np.testing.assert_allclose(allh, one, rtol=1e-14)
    # identical layers -> the layer mean equals one layer
    q_l = np.repeat(q[:1], L, axis=0); k_l = np.repeat(k[:1], L, axis=0)
    np.testing.assert_allclose(oracle.specpc_batch(q_l, k_l, w, 0, 1),
                               oracle.specpc_batch(q_l[:1], k_l[:1], w, 0, 1), rtol=1e-13)
    # skipped layers do not matter
    q2 = q.copy(); q2[0] = rng.standard_normal(q2[0].shape)
    np.testing.assert_array_equal(oracle.specpc_batch(q, k, w, 1, 1),
                                  oracle.specpc_batch(q2, k, w, 1, 1))


def test_specpc_row_weights_endpoints():
    w = W.specpc_row_weights(256)
    assert w[0] == pytest.approx(0.1) and w[-1] == pytest.approx(1.0)
    assert np.all(np.diff(w) > 0)


# ---------------------------------------------------------------- Theorem 1
@pytest.mark.parametrize("eps", [1e-3, 1e-1, 1.0])
def test_theorem1_bound(eps):
    """||s - s_hat||_2 <= eps * ||W_q W_k^T||_2 for unit-norm key embeddings
    (section 关键设计, SpecKV, Theorem 1), on 100 seeds."""
    d_model, d, n_in = 16, 8, 40
    for seed in range(100):
        rng = np.random.default_rng(seed)
        Wq = rng.standard_normal((d_model, d)); Wk = rng.standard_normal((d_model, d))
        X = rng.standard_normal((n_in, d_model)); X /= np.linalg.norm(X, 2)
        x = rng.standard_normal(d_model)
        dx = rng.standard_normal(d_model); dx *= eps / np.linalg.norm(dx)
        q = (x @ Wq)[None, None, :]
        qh = ((x + dx) @ Wq)[None, None, :]
        k = X @ Wk
        s, _ = oracle.speckv_unit(q, k, 0, 1)
        sh, _ = oracle.speckv_unit(qh, k, 0, 1)
        bound = eps * np.linalg.norm(Wq @ Wk.T, 2)
        assert np.linalg.norm(s - sh) <= bound * (1 + 1e-12)


def test_theorem1_bound_summed_rows():
    d_model, d, n_in, R = 12, 8, 30, 6
    rng = np.random.default_rng(99)
    Wq = rng.standard_normal((d_model, d)); Wk = rng.standard_normal((d_model, d))
    X = rng.standard_normal((n_in, d_model)); X /= np.linalg.norm(X, 2)
    x = rng.standard_normal((R, d_model)); dx = 0.05 * rng.standard_normal((R, d_model))
    k = X @ Wk
    s, _ = oracle.speckv_unit((x @ Wq)[None], k, 0, R)
    sh, _ = oracle.speckv_unit(((x + dx) @ Wq)[None], k, 0, R)
    bound = np.linalg.norm(dx, axis=1).sum() * np.linalg.norm(Wq @ Wk.T, 2)
    assert np.linalg.norm(s - sh) <= bound


# ---------------------------------------------------------------- tiny workload
def test_tiny_workload_recovers_planted_keys():
    q, k, v = W.tiny_speckv_numpy(0)
    qb, kb = W.bf16_bits(q), W.bf16_bits(k)
    cfg = W.TINY
    g = cfg.g
    for h in range(cfg.hkv):
        s, p, idx = oracle.speckv_select_unit(qb[0, 0, h * g:(h + 1) * g], kb[0, 0, h],
                                              cfg.n_window, cfg.n_lookahead, cfg.c_max, cfg.pool)
        assert len(idx) == cfg.c_max + cfg.n_window
        sel = set(idx.tolist())
        assert {0, 100, 101, 102, 103} <= sel      # sink and heavy keys are kept
        assert s[0] > np.quantile(s, 0.9)            # the sink ranks high


# ---------------------------------------------------------------- decode attention
def _bf(x):
    return W.bf16_bits(np.asarray(x, np.float32))


def test_decode_single_row_returns_its_value():
    rng = np.random.default_rng(31)
    q = _bf(rng.standard_normal((1, 1, 2, 64)))
    k = _bf(rng.standard_normal((1, 1, 1, 1, 64)))
    v = _bf(rng.standard_normal((1, 1, 1, 1, 64)))
    out = oracle.decode_attention(q, k, v, 0.3)
    np.testing.assert_array_equal(out[0, 0, 0], W.bf16_decode(v)[0, 0, 0, 0].astype(np.float64))
    np.testing.assert_array_equal(out[0, 0, 1], W.bf16_decode(v)[0, 0, 0, 0].astype(np.float64))


def test_decode_identical_keys_average_the_values():
    rng = np.random.default_rng(32)
    q = _bf(rng.standard_normal((1, 1, 1, 64)))
    k = _bf(np.tile(rng.standard_normal((1, 1, 1, 1, 64)), (1, 1, 1, 9, 1)))
    v = _bf(rng.standard_normal((1, 1, 1, 9, 64)))
    out = oracle.decode_attention(q, k, v, 1.0)
    np.testing.assert_allclose(out[0, 0, 0], W.bf16_decode(v)[0, 0, 0].astype(np.float64).mean(0), rtol=0, atol=1e-14)


def test_decode_two_keys_closed_form():
    # z_i = scale * a * b_i exactly (one nonzero coordinate, bf16-exact numbers):
    # out = sigma(z_0 - z_1) v_0 + sigma(z_1 - z_0) v_1
    d = 64
    q = np.zeros((1, 1, 1, d), np.float32); q[..., 5] = 1.5
    k = np.zeros((1, 1, 1, 2, d), np.float32); k[..., 0, 5] = 2.0; k[..., 1, 5] = -0.75
    v = np.zeros((1, 1, 1, 2, d), np.float32); v[..., 0, :] = 3.0; v[..., 1, :] = -1.0
    scale = 0.5
    out = oracle.decode_attention(_bf(q), _bf(k), _bf(v), scale)
    z0, z1 = scale * 1.5 * 2.0, scale * 1.5 * -0.75
    p0 = 1.0 / (1.0 + math.exp(z1 - z0))
    np.testing.assert_allclose(out[0, 0, 0], np.full(d, 3.0 * p0 - (1.0 - p0)), rtol=1e-14)


def test_decode_gqa_heads_read_their_kv_head():
    # KV head 0 holds values +1, KV head 1 values -1: query heads 0, 1 -> +1 and 2, 3 -> -1
    rng = np.random.default_rng(33)
    q = _bf(rng.standard_normal((1, 1, 4, 64)))
    k = _bf(rng.standard_normal((1, 1, 2, 7, 64)))
    v = np.ones((1, 1, 2, 7, 64), np.float32); v[:, :, 1] = -1.0
    out = oracle.decode_attention(q, k, _bf(v), 0.2)
    np.testing.assert_allclose(out[0, 0, :2], 1.0, rtol=1e-14)
    np.testing.assert_allclose(out[0, 0, 2:], -1.0, rtol=1e-14)


def test_decode_row_order_does_not_matter():
    rng = np.random.default_rng(34)
    q = _bf(rng.standard_normal((1, 2, 3, 128)))
    k = _bf(rng.standard_normal((1, 2, 1, 40, 128)))
    v = _bf(rng.standard_normal((1, 2, 1, 40, 128)))
    perm = rng.permutation(40)
    a = oracle.decode_attention(q, k, v, 0.09)
    b = oracle.decode_attention(q, k[:, :, :, perm], v[:, :, :, perm], 0.09)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_decode_dominant_key_wins():
    d = 64
    q = np.zeros((1, 1, 1, d), np.float32); q[..., 0] = 8.0
    k = np.zeros((1, 1, 1, 5, d), np.float32); k[..., 3, 0] = 8.0          # logit 64 vs 0
    v = np.arange(5 * d, dtype=np.float32).reshape(1, 1, 1, 5, d) / 64.0
    out = oracle.decode_attention(_bf(q), _bf(k), _bf(v), 1.0)
    # the other four rows carry weight e^-64 each, |v| <= 5
    np.testing.assert_allclose(out[0, 0, 0], W.bf16_decode(_bf(v))[0, 0, 0, 3], rtol=0, atol=4 * 10 * math.exp(-64))
