"""GPU parity of the prefill attention of the window and lookahead rows
(speckv_prefill_attention) against the fp64 oracle, through the C ABI.

Tolerances, from the arithmetic: the probabilities enter P.V as bf16
(relative rounding <= 2^-9 each) and the output is stored as bf16 (<= 2^-9
of |out|), so |out - ref| <= 2^-8 * max |v| bounds it (fp32 accumulation adds
far less).  The input-key LSE is formed from fp32 probabilities summed in
fp32 over up to tens of thousands of keys: a few 1e-5 in log2 units plus a
few fp32 ulps of |lse2|.  The importance scores that speckv_colsum derives
from the row offsets this attention writes take the scores' 1e-3 bound.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import assert_scores_close, bits_of, to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.load_library()
    P.spk_device_error(clear=True)
    return P


def _case(seed, B, L, hq, hkv, d, n_in, nw, nl, key_gain=1.0):
    rng = np.random.default_rng(seed)
    R = nw + nl
    q = (rng.standard_normal((B, L, hq, R, d)) / math.sqrt(d)).astype(np.float32)
    k = (rng.standard_normal((B, L, hkv, n_in + nl, d)) * key_gain).astype(np.float32)
    v = rng.standard_normal((B, L, hkv, n_in + nl, d)).astype(np.float32)
    u = rng.standard_normal((B, L, hkv, d)).astype(np.float32)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    k[:, :, :, 0] += 4 * u
    heavy = rng.choice(np.arange(1, n_in), size=max(1, n_in // 50), replace=False)
    k[:, :, :, heavy] += 3 * u[:, :, :, None, :]
    q += (1.5 / math.sqrt(d)) * np.repeat(u, hq // hkv, axis=2)[:, :, :, None, :]
    return W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v)


def _run(P, qb, kb, vb, nw, scale=1.0):
    import torch
    B, L, hq, R, d = qb.shape
    hkv, n_kv = kb.shape[2], kb.shape[3]
    nl = R - nw
    n_in = n_kv - nl
    q = to_bf16_tensor(qb)
    k = to_bf16_tensor(np.ascontiguousarray(kb[:, :, :, :n_in]))
    v = to_bf16_tensor(np.ascontiguousarray(vb[:, :, :, :n_in]))
    kl = to_bf16_tensor(np.ascontiguousarray(kb[:, :, :, n_in:])) if nl else None
    vl = to_bf16_tensor(np.ascontiguousarray(vb[:, :, :, n_in:])) if nl else None
    units, g = B * L * hkv, hq // hkv
    lse2 = torch.empty((units, g * R), dtype=torch.float32, device="cuda")
    shape = P.binding.speckv_shape(q, k, nw, scale)
    ws = torch.empty(P.speckv_workspace_size(shape), dtype=torch.uint8, device="cuda")
    out = P.speckv_prefill_attention(q, k, v, kl, vl, nw, lse2=lse2, workspace=ws, scale=scale)
    scores = torch.empty((units, n_in - nw), dtype=torch.float32, device="cuda") if n_in > nw else None
    if scores is not None:
        P.speckv_colsum(q, k, nw, scores, ws, scale=scale)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    return out, lse2, scores, (q, k, v, kl, vl, ws)


def _check(P, qb, kb, vb, nw, scale=1.0):
    B, L, hq, R, d = qb.shape
    hkv, n_kv = kb.shape[2], kb.shape[3]
    nl = R - nw
    n_in = n_kv - nl
    g = hq // hkv
    out, lse2, scores, _ = _run(P, qb, kb, vb, nw, scale)
    ob = W.bf16_decode(bits_of(out)).astype(np.float64)
    lse = lse2.cpu().numpy()
    sc = scores.cpu().numpy() if scores is not None else None
    for u in range(B * L * hkv):
        b, l, h = u // (L * hkv), (u // hkv) % L, u % hkv
        qu, ku, vu = qb[b, l, h * g:(h + 1) * g], kb[b, l, h], vb[b, l, h]
        ref, rlse = oracle.prefill_unit(qu, ku, vu, nw, nl, n_in, scale)
        vmax = np.abs(W.bf16_decode(vu)).max()
        err = np.abs(ob[b, l, h * g:(h + 1) * g] - ref).max()
        assert err <= 2.0 ** -8 * vmax, f"unit {u}: out error {err:.3e} > {2.0 ** -8 * vmax:.3e}"
        l2 = rlse / math.log(2.0)
        np.testing.assert_allclose(lse[u], l2, rtol=4e-7, atol=6e-5)
        if sc is not None:
            s, _ = oracle.speckv_unit(qu, ku[:n_in], nw, nl, scale)
            assert_scores_close(sc[u], s, f"scores from the prefill's row offsets, unit {u}")


@pytest.mark.parametrize("case", [
    # seed, B, L, hq, hkv, d, n_in, n_window, n_lookahead
    (1, 1, 2, 4, 2, 128, 700, 16, 16),      # ragged input tiles, one lookahead tile
    (2, 1, 1, 6, 2, 64, 1000, 40, 24),      # head_dim 64
    (3, 2, 1, 10, 2, 128, 513, 64, 128),    # 960 rows (8 row tiles), a full lookahead tile
    (4, 1, 1, 4, 2, 128, 300, 32, 0),       # no lookahead: window rows only
    (5, 1, 1, 2, 1, 64, 129, 0, 200),       # no window; two lookahead tiles (the second ragged)
    (6, 1, 1, 4, 4, 128, 96, 96, 4),        # window covers the whole input
    (7, 1, 1, 16, 1, 128, 1500, 64, 64),    # g * R = 2048 rows
    (10, 1, 1, 6, 2, 128, 800, 60, 60),     # 360 rows: three Q tiles, the second pair's B tile empty
])
def test_prefill_attention_parity(P, case):
    seed, B, L, hq, hkv, d, n_in, nw, nl = case
    qb, kb, vb = _case(seed, B, L, hq, hkv, d, n_in, nw, nl)
    _check(P, qb, kb, vb, nw)


def test_prefill_attention_rescales(P):
    # logits spanning tens of powers of two, and the largest ones late in the
    # sequence: the running maximum moves several times (lazy rescale of O)
    qb, kb, vb = _case(8, 1, 1, 4, 2, 128, 900, 32, 32, key_gain=6.0)
    k = W.bf16_decode(kb)
    k[..., 850:, :] *= 2.0
    _check(P, qb, W.bf16_bits(k), vb, 32, scale=0.8)


def test_prefill_attention_deterministic(P):
    import torch
    qb, kb, vb = _case(9, 1, 2, 8, 2, 128, 1200, 32, 32)
    a, la, sa, _ = _run(P, qb, kb, vb, 32)
    b, lb, sb, _ = _run(P, qb, kb, vb, 32)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb) and torch.equal(sa, sb)
