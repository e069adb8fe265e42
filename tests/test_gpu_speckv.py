"""GPU parity of the SpecKV path (scores -> pool + top-k + window -> compaction)
against the fp64 oracle, through the C ABI (prompt_compression_b200.binding).

Small cases run the oracle on every unit: they span several 128-key and
128-row tiles, ragged tails, GQA groups, and the degenerate settings of the
method (no lookahead = SnapKV-style scoring, no window, window = whole input,
C_max >= n_pre).
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import (assert_indices_match, assert_scores_close, bits_of, oracle_unit,
                               to_bf16_tensor)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import torch  # noqa: F401
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.load_library()
    P.spk_device_error(clear=True)
    return P


def _random_case(seed, B, L, hq, hkv, d, n_in, n_window, n_lookahead, planted=True):
    rng = np.random.default_rng(seed)
    R = n_window + n_lookahead
    q = rng.standard_normal((B, L, hq, R, d)).astype(np.float32)
    k = rng.standard_normal((B, L, hkv, n_in, d)).astype(np.float32)
    v = rng.standard_normal((B, L, hkv, n_in, d)).astype(np.float32)
    if planted:
        u = rng.standard_normal((B, L, hkv, d)).astype(np.float32)
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        k[:, :, :, 0] += 4 * u
        heavy = rng.choice(np.arange(1, max(n_in - n_window, 2)), size=max(1, n_in // 50), replace=False)
        k[:, :, :, heavy] += 3 * u[:, :, :, None, :]
        q += 1.5 * np.repeat(u, hq // hkv, axis=2)[:, :, :, None, :]
    q /= math.sqrt(d)
    return W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v)


def _run_and_check(P, qb, kb, vb, n_window, c_max, pool=7, scale=1.0):
    import torch
    B, L, hq, R, d = qb.shape
    hkv, n_in = kb.shape[2], kb.shape[3]
    g = hq // hkv
    n_lookahead = R - n_window
    q, k, v = to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb)
    buf = P.pipeline.SpeckvBuffers(q, k, v, n_window, c_max, window_mass=n_window > 0, with_pooled=True)
    P.speckv_compress(q, k, v, n_window, c_max, pool, scale, buffers=buf)
    lse2 = torch.empty((buf.units, g * R), dtype=torch.float32, device="cuda")
    P.speckv_row_lse(q, k, n_window, lse2, scale)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    scores = buf.scores.cpu().numpy()
    pooled = buf.pooled.cpu().numpy()
    wmass = buf.window_mass.cpu().numpy() if buf.window_mass is not None else None
    idx = buf.idx.cpu().numpy()
    lse = lse2.cpu().numpy()
    k_out, v_out = bits_of(buf.k_out), bits_of(buf.v_out)
    n_pre = n_in - n_window
    c = min(c_max, n_pre)
    for u in range(buf.units):
        b, l, h = u // (L * hkv), (u // hkv) % L, u % hkv
        qu = qb[b, l, h * g:(h + 1) * g]
        ku = kb[b, l, h]
        s, wm, p, ridx = oracle_unit(qu, ku, n_window, n_lookahead, c_max, pool, scale)
        _, _, olse = oracle.speckv_unit(qu, ku, n_window, n_lookahead, scale, with_lse=True)
        # pass 1: log2-domain LSE of every row; fp32 logits and the fp32 sum
        # M + log2(L) carry a few ulps of |lse2| on top of the absolute part
        np.testing.assert_allclose(lse[u], olse / math.log(2.0), rtol=4e-7, atol=2e-5)
        assert_scores_close(scores[u], s, f"scores[{u}]")
        if wmass is not None:
            assert_scores_close(wmass[u], wm, f"window_mass[{u}]")
            # every row's softmax sums to 1: columns sum to g * R
            tot = scores[u].astype(np.float64).sum() + wmass[u].astype(np.float64).sum()
            assert abs(tot - g * R) < 1e-4 * g * R
        # pooling is exact; selection is bit-exact on the GPU's own scores
        np.testing.assert_array_equal(pooled[u], oracle.maxpool(scores[u].astype(np.float64), pool)
                                      .astype(np.float32))
        own = oracle.topk_with_tail(scores[u].astype(np.float64) if pool == 1 else
                                    oracle.maxpool(scores[u].astype(np.float64), pool), c_max, n_window)
        assert np.array_equal(idx[u], own), f"unit {u}: selection differs from the oracle on the same scores"
        assert_indices_match(idx[u], ridx, p, c)
        # compaction: bit-exact rows at the GPU's indices
        np.testing.assert_array_equal(k_out[b, l, h], kb[b, l, h][idx[u]])
        np.testing.assert_array_equal(v_out[b, l, h], vb[b, l, h][idx[u]])
    return buf


def test_tiny_workload(P):
    q, k, v = W.tiny_speckv_numpy(0)
    cfg = W.TINY
    buf = _run_and_check(P, W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), cfg.n_window, cfg.c_max, cfg.pool)
    idx = buf.idx.cpu().numpy()
    for u in range(buf.units):
        assert {0, 100, 101, 102, 103} <= set(idx[u].tolist())


@pytest.mark.parametrize("case", [
    # seed, B, L, hq, hkv, d, n_in, n_window, n_lookahead, c_max
    (1, 1, 2, 6, 2, 128, 1000, 40, 24, 100),     # ragged key tail, g=3, 192 rows
    (2, 2, 1, 10, 2, 128, 700, 64, 32, 64),      # 480 rows: two row blocks, half-empty tile
    (3, 1, 1, 4, 4, 64, 300, 0, 16, 32),         # no window
    (4, 1, 1, 8, 2, 64, 513, 32, 0, 128),        # no lookahead (SnapKV-style)
    (5, 1, 1, 2, 1, 128, 129, 16, 8, 500),       # C_max >= n_pre keeps everything
    (6, 1, 1, 4, 2, 64, 96, 96, 4, 8),           # window covers the whole input
    (7, 1, 3, 5, 1, 128, 2100, 64, 128, 256),    # Qwen-like group: 960 rows, 7.5 row tiles
    (8, 1, 1, 16, 1, 128, 1500, 64, 64, 200),    # g * R = 2048 rows: the largest unit
    (9, 1, 1, 32, 2, 64, 777, 48, 80, 64),       # g * R = 2048 with head_dim 64, ragged keys
])
def test_speckv_shapes(P, case):
    seed, B, L, hq, hkv, d, n_in, nw, nl, c_max = case
    qb, kb, vb = _random_case(seed, B, L, hq, hkv, d, n_in, nw, nl)
    _run_and_check(P, qb, kb, vb, nw, c_max)


def test_scale_argument(P):
    qb, kb, vb = _random_case(11, 1, 1, 4, 2, 64, 400, 16, 16)
    _run_and_check(P, qb, kb, vb, 16, 64, scale=0.61)


@pytest.mark.parametrize("key_gain,scale", [(24.0, 0.05), (6.0, 4.0)])
def test_large_logits_and_normalisers(P, key_gain, scale):
    # The column pass adds each row's -lse2/c2 to the accumulator as three
    # bf16 terms: q.k of magnitude ~100 against a small scale, and logits
    # spanning tens of powers of two, both have to come out at the
    # oracle's scores.
    qb, kb, vb = _random_case(13, 1, 2, 6, 2, 128, 900, 32, 32)
    k = W.bf16_decode(kb) * key_gain
    _run_and_check(P, qb, W.bf16_bits(k), vb, 32, 96, scale=scale)


def test_pool_kernel_one_and_three(P):
    qb, kb, vb = _random_case(12, 1, 1, 4, 2, 64, 333, 8, 8)
    _run_and_check(P, qb, kb, vb, 8, 40, pool=1)
    _run_and_check(P, qb, kb, vb, 8, 40, pool=3)


def test_deterministic(P):
    import torch
    qb, kb, vb = _random_case(13, 1, 2, 8, 2, 128, 1500, 32, 32)
    q, k, v = to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb)
    a = P.speckv_compress(q, k, v, 32, 128, 7, window_mass=True)
    sa, ia, ka = a.scores.clone(), a.idx.clone(), a.k_out.clone()
    b = P.speckv_compress(q, k, v, 32, 128, 7, window_mass=True)
    torch.cuda.synchronize()
    assert torch.equal(sa, b.scores) and torch.equal(ia, b.idx) and torch.equal(ka, b.k_out)


def test_split_passes_equal_speckv_score(P):
    # speckv_score is speckv_row_offsets then speckv_colsum: bit for bit
    import torch
    qb, kb, vb = _random_case(29, 1, 2, 8, 2, 128, 1300, 32, 64)
    q, k = to_bf16_tensor(qb), to_bf16_tensor(kb)
    units, n_pre = 4, 1300 - 32
    a = torch.empty((units, n_pre), dtype=torch.float32, device="cuda")
    wa = torch.empty((units, 32), dtype=torch.float32, device="cuda")
    P.speckv_score(q, k, 32, a, wa)
    ws = torch.empty(P.speckv_workspace_size(P.binding.speckv_shape(q, k, 32)), dtype=torch.uint8, device="cuda")
    b = torch.full_like(a, float("nan"))
    wb = torch.full_like(wa, float("nan"))
    P.speckv_row_offsets(q, k, 32, ws)
    P.speckv_colsum(q, k, 32, b, ws, window_mass=wb)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(wa, wb)


def test_uniform_keys_ties_lowest_index(P):
    # identical keys: all prefix scores tie exactly -> indices 0..C-1
    import torch
    rng = np.random.default_rng(14)
    d, n_in, nw, nl = 64, 640, 16, 16
    q = (rng.standard_normal((1, 1, 4, nw + nl, d)) / 8).astype(np.float32)
    k = np.tile(rng.standard_normal((1, 1, 2, 1, d)).astype(np.float32), (1, 1, 1, n_in, 1))
    qb, kb = W.bf16_bits(q), W.bf16_bits(k)
    buf = P.speckv_compress(to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(kb), nw, 64, 7)
    torch.cuda.synchronize()
    idx = buf.idx.cpu().numpy()
    for u in range(2):
        assert idx[u].tolist() == list(range(64)) + list(range(n_in - nw, n_in))


def test_topk_select_direct(P):
    """topk_select alone on integer-valued scores (many exact ties), bit-exact."""
    import torch
    rng = np.random.default_rng(15)
    for n, kk, tail, pool in [(5000, 300, 7, 7), (65472, 256, 64, 7), (100, 0, 5, 3), (37, 50, 0, 1),
                              (2, 1, 0, 7), (0, 4, 3, 7)]:
        s = rng.integers(0, 20, size=(3, n)).astype(np.float32) * 0.25
        st = torch.from_numpy(s).cuda()
        c = min(kk, n)
        idx = torch.empty((3, c + tail), dtype=torch.int32, device="cuda")
        P.topk_select(st, kk, tail, idx, pool)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        for u in range(3):
            ref = oracle.topk_with_tail(oracle.maxpool(s[u].astype(np.float64), pool) if n else
                                        np.zeros(0), kk, tail)
            assert got[u].tolist() == ref.tolist(), (n, kk, tail, pool)


@pytest.mark.parametrize("mode", ["max", "avg"])
def test_topk_paths_on_continuous_scores(P, mode):
    """Selection on continuous scores (C from 1 to above 2048, rows split
    over one to four CTAs, pooling radius 0 to 511) with either pooling;
    bit-exact against the oracle's selection on the GPU's own pooled values,
    which match the oracle's pooling of the GPU's scores (max: exactly; avg:
    an fp32 sum of `pool` terms and one division, within (pool + 1) * 2^-24
    relative)."""
    import torch
    rng = np.random.default_rng(19)
    pm = P.SPK_POOL_MAX if mode == "max" else P.SPK_POOL_AVG
    for n, kk, tail, pool in [(65472, 256, 64, 7), (65472, 2048, 0, 7), (65472, 2049, 0, 7),
                              (20000, 5000, 3, 3), (777, 1, 2, 9), (777, 776, 0, 1), (4096, 300, 0, 1023),
                              (30000, 77, 0, 9)]:
        s = (rng.gamma(2.0, 1.0, size=(3, n)) * rng.random((3, 1))).astype(np.float32)
        st = torch.from_numpy(s).cuda()
        c = min(kk, n)
        idx = torch.empty((3, c + tail), dtype=torch.int32, device="cuda")
        pooled = torch.empty((3, n), dtype=torch.float32, device="cuda")
        P.topk_select(st, kk, tail, idx, pool, pooled=pooled, pool_mode=pm)
        torch.cuda.synchronize()
        got, gp = idx.cpu().numpy(), pooled.cpu().numpy()
        for u in range(3):
            ref_pool = oracle.pool(s[u].astype(np.float64), pool, mode)
            if mode == "max":
                np.testing.assert_array_equal(gp[u], ref_pool.astype(np.float32))
            else:
                # fp32 sum of `pool` non-negative terms then one rounded
                # division: relative error <= (pool + 1) * 2^-24
                np.testing.assert_allclose(gp[u], ref_pool, rtol=(pool + 1) * 2.0 ** -24, atol=0)
            own = oracle.topk_with_tail(gp[u].astype(np.float64), kk, tail)
            assert got[u].tolist() == own.tolist(), (n, kk, tail, pool, mode)
    assert P.spk_device_error() == (0, 0)


def test_topk_refines_a_crowded_bin(P):
    """Scores in [1, 1.1) share one 12-bit key bin (sign, exponent, three
    mantissa bits): the selection refines it by the next 12 and then the last
    8 bits; bit-exact against the oracle on the same values."""
    import torch
    rng = np.random.default_rng(37)
    for n, kk, tail, pool in [(65472, 256, 64, 7), (30000, 2048, 0, 1), (9999, 700, 5, 3)]:
        s = (1.0 + 0.1 * rng.random((2, n))).astype(np.float32)
        st = torch.from_numpy(s).cuda()
        idx = torch.empty((2, min(kk, n) + tail), dtype=torch.int32, device="cuda")
        P.topk_select(st, kk, tail, idx, pool)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        for u in range(2):
            ref = oracle.topk_with_tail(oracle.maxpool(s[u].astype(np.float64), pool), kk, tail)
            assert got[u].tolist() == ref.tolist(), (n, kk, tail, pool)
    assert P.spk_device_error() == (0, 0)


@pytest.mark.parametrize("mode", ["max", "avg"])
def test_topk_row_layouts(P, mode):
    """Every way a row is laid out: one CTA (n <= 16384), clusters of 2, 4 and
    8 CTAs (two CTAs per SM), eight CTAs of up to 40960 candidates (one per
    SM), and the workspace kernel (longer rows, or a pooling radius beyond
    1024); pooling radii inside and past the unrolled windows.  Integer-valued
    scores, so ties straddle the CTA boundaries; bit-exact selection against
    the oracle on the GPU's own pooled values."""
    import torch
    rng = np.random.default_rng(41)
    pm = P.SPK_POOL_MAX if mode == "max" else P.SPK_POOL_AVG
    for n, kk, tail, pool in [(16384, 1000, 4, 5), (16385, 1000, 0, 13), (40000, 3000, 2, 15),
                              (100000, 5000, 3, 7), (131072, 257, 0, 1), (200000, 3000, 0, 11),
                              (327680, 100, 1, 3), (327681, 100, 1, 3), (400000, 6000, 0, 7),
                              (5000, 300, 1, 2049), (70000, 700, 0, 513)]:
        s = rng.integers(0, 40, size=(2, n)).astype(np.float32) * 0.125
        st = torch.from_numpy(s).cuda()
        c = min(kk, n)
        idx = torch.empty((2, c + tail), dtype=torch.int32, device="cuda")
        pooled = torch.empty((2, n), dtype=torch.float32, device="cuda")
        P.topk_select(st, kk, tail, idx, pool, pooled=pooled, pool_mode=pm)
        torch.cuda.synchronize()
        got, gp = idx.cpu().numpy(), pooled.cpu().numpy()
        for u in range(2):
            ref_pool = oracle.pool(s[u].astype(np.float64), pool, mode)
            if mode == "max":
                np.testing.assert_array_equal(gp[u], ref_pool.astype(np.float32))
            else:
                np.testing.assert_allclose(gp[u], ref_pool, rtol=(pool + 1) * 2.0 ** -24, atol=0)
            own = oracle.topk_with_tail(gp[u].astype(np.float64), kk, tail)
            assert got[u].tolist() == own.tolist(), (n, kk, tail, pool, mode)
    assert P.spk_device_error() == (0, 0)


def test_topk_degenerate_counts_on_clusters(P):
    """C = 0 (the window only, with the pooled output requested) and C >= n
    (every candidate) on rows split over clusters of 2, 4 and 8 CTAs."""
    import torch
    rng = np.random.default_rng(43)
    for n, kk, tail, pool in [(40000, 0, 5, 7), (100000, 0, 0, 3), (50000, 50000, 3, 5), (200000, 250000, 2, 7)]:
        s = rng.random((2, n)).astype(np.float32)
        st = torch.from_numpy(s).cuda()
        c = min(kk, n)
        idx = torch.empty((2, c + tail), dtype=torch.int32, device="cuda")
        pooled = torch.empty((2, n), dtype=torch.float32, device="cuda")
        P.topk_select(st, kk, tail, idx, pool, pooled=pooled)
        torch.cuda.synchronize()
        got, gp = idx.cpu().numpy(), pooled.cpu().numpy()
        for u in range(2):
            np.testing.assert_array_equal(gp[u], oracle.maxpool(s[u].astype(np.float64), pool).astype(np.float32))
            assert got[u].tolist() == list(range(c)) + list(range(n, n + tail)), (n, kk, tail)
    assert P.spk_device_error() == (0, 0)


def test_speckv_avg_pool_end_to_end(P):
    """speckv_compress with average pooling: scores against the oracle, the
    selection bit-exact on the GPU's own pooled values and tie-tolerant
    against the oracle's own average-pooled selection."""
    import torch
    qb, kb, vb = _random_case(23, 1, 2, 8, 2, 128, 1500, 32, 32)
    q, k, v = to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb)
    buf = P.pipeline.SpeckvBuffers(q, k, v, 32, 128, with_pooled=True)
    P.speckv_compress(q, k, v, 32, 128, 5, buffers=buf, pool_mode=P.SPK_POOL_AVG)
    torch.cuda.synchronize()
    scores, pooled, idx = buf.scores.cpu().numpy(), buf.pooled.cpu().numpy(), buf.idx.cpu().numpy()
    kout = bits_of(buf.k_out)
    for u in range(buf.units):
        l, h = u // 2, u % 2
        s, _ = oracle.speckv_unit(qb[0, l, h * 4:(h + 1) * 4], kb[0, l, h], 32, 32)
        assert_scores_close(scores[u], s, f"scores[{u}]")
        np.testing.assert_allclose(pooled[u], oracle.avgpool(scores[u].astype(np.float64), 5), rtol=6 * 2.0 ** -24,
                                   atol=0)
        assert idx[u].tolist() == oracle.topk_with_tail(pooled[u].astype(np.float64), 128, 32).tolist()
        p = oracle.avgpool(s, 5)
        assert_indices_match(idx[u], oracle.topk_with_tail(p, 128, 32), p, 128)
        np.testing.assert_array_equal(kout[0, l, h], kb[0, l, h][idx[u]])


def test_kv_compact_broadcast_and_errors(P):
    import torch
    rng = np.random.default_rng(16)
    units, n_src, d = 6, 300, 64
    kb = rng.integers(0, 2 ** 16, size=(units, n_src, d), dtype=np.uint16)
    vb = rng.integers(0, 2 ** 16, size=(units, n_src, d), dtype=np.uint16)
    idx = np.stack([np.sort(rng.choice(n_src, 40, replace=False)) for _ in range(2)]).astype(np.int32)
    k, v = to_bf16_tensor(kb), to_bf16_tensor(vb)
    ko = torch.empty((units, 40, d), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    P.kv_compact(k, v, torch.from_numpy(idx).cuda(), ko, vo, units_per_idx=3)
    torch.cuda.synchronize()
    ko_b, vo_b = bits_of(ko), bits_of(vo)
    for u in range(units):
        np.testing.assert_array_equal(ko_b[u], kb[u][idx[u // 3]])
        np.testing.assert_array_equal(vo_b[u], vb[u][idx[u // 3]])
    assert P.spk_device_error() == (0, 0)
    bad = idx.copy()
    bad[1, 5] = n_src     # out of range: recorded, row left unwritten, nothing faults
    P.kv_compact(k, v, torch.from_numpy(bad).cuda(), ko, vo, units_per_idx=3)
    st, site = P.spk_device_error()
    assert st == P.binding.SPK_ERR_ARG
    assert P.spk_device_error() == (0, 0)


def test_kv_compact_from_pinned_host_memory(P):
    # K on the device, V left in page-locked host memory: the gather reads
    # only the selected V rows in place and matches the device-resident copy
    import torch
    rng = np.random.default_rng(17)
    units, n_src, d, n_idx = 4, 500, 128, 64
    kb = rng.integers(0, 2 ** 16, size=(units, n_src, d), dtype=np.uint16)
    vb = rng.integers(0, 2 ** 16, size=(units, n_src, d), dtype=np.uint16)
    idx = np.stack([np.sort(rng.choice(n_src, n_idx, replace=False)) for _ in range(units)]).astype(np.int32)
    k = to_bf16_tensor(kb)
    vh = to_bf16_tensor(vb, device="cpu").pin_memory()
    ko = torch.empty((units, n_idx, d), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    P.kv_compact(k, vh, torch.from_numpy(idx).cuda(), ko, vo)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    ko_b, vo_b = bits_of(ko), bits_of(vo)
    for u in range(units):
        np.testing.assert_array_equal(ko_b[u], kb[u][idx[u]])
        np.testing.assert_array_equal(vo_b[u], vb[u][idx[u]])
    # pageable host memory is refused before anything is launched
    with pytest.raises(ValueError):
        P.kv_compact(k, to_bf16_tensor(vb, device="cpu"), torch.from_numpy(idx).cuda(), ko, vo)


def test_argument_errors_do_not_launch(P):
    import torch
    q = torch.zeros((1, 1, 4, 8, 96), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 2, 64, 96), dtype=torch.bfloat16, device="cuda")
    s = torch.zeros((2, 60), dtype=torch.float32, device="cuda")
    with pytest.raises(P.SpeckvError) as e:
        P.speckv_score(q, k, 4, s)
    assert e.value.status == P.binding.SPK_ERR_UNSUPPORTED
    q = torch.zeros((1, 1, 4, 8, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 3, 64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(P.SpeckvError) as e:      # 3 KV heads: the shape is rejected by the library
        P.speckv_score(q, k, 4, torch.zeros((3, 60), dtype=torch.float32, device="cuda"))
    assert e.value.status == P.binding.SPK_ERR_ARG
    k = torch.zeros((1, 1, 2, 64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(P.SpeckvError) as e:
        P.speckv_score(q, k, 4, s, workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == P.binding.SPK_ERR_WORKSPACE
    assert P.spk_device_error() == (0, 0)
