"""GPU parity of SpecPC scoring and selection, and of the SpecKV-PC cascade,
against the fp64 oracle through the C ABI."""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import assert_indices_match, assert_scores_close, bits_of, to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.load_library()
    P.spk_device_error(clear=True)
    return P


def _case(seed, B, L, hq, hkv, d, n_in, Wr):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((B, L, hq, Wr, d)) / math.sqrt(d)).astype(np.float32)
    k = rng.standard_normal((B, L, hkv, n_in, d)).astype(np.float32)
    u = rng.standard_normal((B, L, hkv, d)).astype(np.float32)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    heavy = rng.choice(np.arange(1, n_in), size=max(1, n_in // 100), replace=False)
    k[:, :, :, heavy] += 3 * u[:, :, :, None, :]
    q += (1.5 / math.sqrt(d)) * np.repeat(u, hq // hkv, axis=2)[:, :, :, None, :]
    return W.bf16_bits(q), W.bf16_bits(k)


def _check_specpc(P, seed, B, L, l_skip, hq, hkv, n_in, Wr, nl, keep, d, w=None):
    import torch
    qb, kb = _case(seed, B, L, hq, hkv, d, n_in, Wr)
    w = W.specpc_row_weights(Wr) if w is None else w
    q, k = to_bf16_tensor(qb), to_bf16_tensor(kb)
    wt = torch.from_numpy(w.astype(np.float32)).cuda()
    scores, idx = P.specpc_select(q, k, wt, l_skip, keep, 7, n_lookahead=nl)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    s_gpu = scores.cpu().numpy()
    i_gpu = idx.cpu().numpy()
    assert np.isfinite(s_gpu).all()
    refs = []
    for b in range(B):
        ref = oracle.specpc_batch(qb[b], kb[b], w.astype(np.float32).astype(np.float64), l_skip, nl)
        assert_scores_close(s_gpu[b], ref, f"specpc scores[{b}]")
        p = oracle.maxpool(ref, 7)
        ridx = oracle.topk_with_tail(p, keep, 0)
        own = oracle.topk_with_tail(oracle.maxpool(s_gpu[b].astype(np.float64), 7), keep, 0)
        assert np.array_equal(i_gpu[b], own)
        assert_indices_match(i_gpu[b], ridx, p, min(keep, n_in))
        refs.append(ref)
    return s_gpu, refs


@pytest.mark.parametrize("case", [
    # seed, B, L, l_skip, hq, hkv, n_in, W, n_lookahead, keep
    (1, 1, 3, 1, 4, 2, 700, 64, 1, 100),
    (2, 2, 2, 0, 6, 2, 333, 40, 1, 50),      # W not a multiple of 32: groups straddle query heads
    (3, 1, 4, 3, 7, 1, 1030, 256, 1, 200),   # g = 7 query heads of 256 rows (draft-like)
    (4, 1, 2, 1, 2, 2, 257, 17, 3, 64),      # lookahead > 1: rows past the input see every key
    (5, 1, 2, 1, 32, 4, 600, 256, 1, 80),    # 32 query heads (the most), g * W = 2048 rows
])
def test_specpc_parity(P, case):
    _check_specpc(P, *case, d=64)


@pytest.mark.parametrize("case", [
    # seed, B, L, l_skip, hq, hkv, n_in, W, n_lookahead, keep -- head_dim 128 drafts
    (11, 1, 3, 1, 4, 2, 700, 64, 1, 100),
    (12, 2, 2, 0, 6, 2, 333, 40, 1, 50),     # W not a multiple of 32, ragged keys
    (13, 1, 3, 1, 12, 2, 1030, 256, 1, 200), # a 1.5B-class draft: 12 / 2 heads, g * W = 1536 rows
    (14, 1, 2, 1, 32, 4, 600, 256, 1, 80),   # 32 query heads, g * W = 2048 rows
    (15, 1, 2, 1, 2, 2, 257, 17, 3, 64),     # lookahead > 1
])
def test_specpc_parity_head_dim_128(P, case):
    _check_specpc(P, *case, d=128)


@pytest.mark.parametrize("d", [64, 128])
def test_specpc_zero_row_weights(P, d):
    # rows of weight 0 add nothing; the last rows (the only ones that see the
    # last keys) are among them, so those keys score exactly 0 in the oracle
    Wr, n_in = 48, 500
    w = W.specpc_row_weights(Wr)
    w[::3] = 0.0
    w[-5:] = 0.0
    s_gpu, refs = _check_specpc(P, 21 + d, 1, 3, 1, 6, 2, n_in, Wr, 1, 60, d, w=w)
    assert (refs[0][-4:] == 0.0).all()
    assert np.abs(s_gpu[0][-4:]).max() <= 1e-30


@pytest.mark.parametrize("d", [64, 128])
def test_specpc_split_passes_equal_specpc_score(P, d):
    # specpc_score is specpc_row_offsets then specpc_colsum, bit for bit, and
    # repeated calls give the same bits (with and without segment groups)
    import torch
    for L, l_skip, hkv in ((4, 1, 2), (2, 1, 1)):      # 6 segments (grouped) and 1 segment
        qb, kb = _case(31 + L, 1, L, 2 * hkv, hkv, d, 900, 64)
        q, k = to_bf16_tensor(qb), to_bf16_tensor(kb)
        wt = torch.from_numpy(W.specpc_row_weights(64).astype(np.float32)).cuda()
        a = torch.empty((1, 900), dtype=torch.float32, device="cuda")
        P.specpc_score(q, k, wt, a, l_skip)
        shape = P.binding.specpc_shape(q, k, l_skip, 1)
        ws = torch.empty(P.specpc_workspace_size(shape), dtype=torch.uint8, device="cuda")
        b = torch.full_like(a, float("nan"))
        P.specpc_row_offsets(q, k, wt, ws, l_skip)
        P.specpc_colsum(q, k, b, ws, l_skip)
        c = torch.full_like(a, float("nan"))
        P.specpc_score(q, k, wt, c, l_skip, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(a, b) and torch.equal(a, c)


def test_cascade_small(P):
    """SpecPC keeps 256 of 1500 tokens; the target K/V are gathered there and
    SpecKV keeps 32 + window of the gathered cache."""
    import torch
    rng = np.random.default_rng(21)
    B, Ld, n_in, keep = 1, 3, 1500, 256
    qd, kd = _case(22, B, Ld, 4, 2, 64, n_in, 64)
    Lt, hq, hkv, d, nw, nl, c_max = 2, 4, 2, 128, 16, 16, 32
    kt = W.bf16_bits(rng.standard_normal((B, Lt, hkv, n_in, d)).astype(np.float32))
    vt = W.bf16_bits(rng.standard_normal((B, Lt, hkv, n_in, d)).astype(np.float32))
    qt = W.bf16_bits((rng.standard_normal((B, Lt, hq, nw + nl, d)) / math.sqrt(d)).astype(np.float32))
    w = W.specpc_row_weights(64).astype(np.float32)
    pc_scores, pc_idx, k_g, v_g, out = P.cascade_compress(
        to_bf16_tensor(qd), to_bf16_tensor(kd), torch.from_numpy(w).cuda(), 1, keep,
        to_bf16_tensor(qt), to_bf16_tensor(kt), to_bf16_tensor(vt), nw, c_max)
    torch.cuda.synchronize()
    pidx = pc_idx.cpu().numpy()
    kg, vg = bits_of(k_g), bits_of(v_g)
    for l in range(Lt):
        for h in range(hkv):
            np.testing.assert_array_equal(kg[0, l, h], kt[0, l, h][pidx[0]])
            np.testing.assert_array_equal(vg[0, l, h], vt[0, l, h][pidx[0]])
    # step 2 is SpecKV on the gathered cache
    idx2 = out.idx.cpu().numpy()
    s2 = out.scores.cpu().numpy()
    g = hq // hkv
    for u in range(Lt * hkv):
        l, h = u // hkv, u % hkv
        s, wm = oracle.speckv_unit(qt[0, l, h * g:(h + 1) * g], kg[0, l, h], nw, nl)
        assert_scores_close(s2[u], s, f"cascade step-2 scores[{u}]")
        p = oracle.maxpool(s, 7)
        assert_indices_match(idx2[u], oracle.topk_with_tail(p, c_max, nw), p, c_max)
