"""GPU parity of the Vertical-Slash sparse prefill attention
(vs_sparse_attention) against the fp64 oracle, through the C ABI.

Tolerances as for the prefill attention: probabilities enter P.V as bf16 and
the output is stored as bf16, so |out - ref| <= 2^-8 * max |v|; the LSE is
formed in fp32 from fp32 probabilities (a few 1e-5 in log2 units plus a few
fp32 ulps of |lse2|)."""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import bits_of, to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.load_library()
    P.spk_device_error(clear=True)
    return P


def _pattern(rng, units, n, n_v, n_s, local=16):
    """Per unit: vertical columns (the sink plus random keys) and slash
    offsets (the local window plus random far diagonals), ascending."""
    vert, sl = [], []
    for _ in range(units):
        v = set([0] if n_v else []) | set(rng.choice(n, size=max(0, n_v - 1), replace=False).tolist())
        while len(v) < n_v:
            v.add(int(rng.integers(0, n)))
        s = set(range(min(local, n_s, n)))
        while len(s) < n_s:
            s.add(int(rng.integers(0, n)))
        vert.append(sorted(v)[:n_v])
        sl.append(sorted(s)[:n_s])
    return np.array(vert, np.int32).reshape(units, n_v), np.array(sl, np.int32).reshape(units, n_s)


def _run(P, qb, kb, vb, vert, sl, scale=1.0):
    import torch
    q, k, v = to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb)
    B, L, hq, n_q, d = qb.shape
    lse2 = torch.empty((B * L * hq, n_q), dtype=torch.float32, device="cuda")
    out = P.vs_sparse_attention(q, k, v, torch.from_numpy(vert).cuda(), torch.from_numpy(sl).cuda(), lse2=lse2,
                                scale=scale)
    torch.cuda.synchronize()
    return out, lse2


def _check(P, qb, kb, vb, vert, sl, scale=1.0):
    B, L, hq, n_q, d = qb.shape
    hkv = kb.shape[2]
    g = hq // hkv
    out, lse2 = _run(P, qb, kb, vb, vert, sl, scale)
    assert P.spk_device_error() == (0, 0)
    ob = W.bf16_decode(bits_of(out)).astype(np.float64)
    lse = lse2.cpu().numpy()
    for u in range(B * L * hkv):
        b, l, h = u // (L * hkv), (u // hkv) % L, u % hkv
        ref, rlse = oracle.vs_attention_unit(qb[b, l, h * g:(h + 1) * g], kb[b, l, h], vb[b, l, h], vert[u], sl[u],
                                             scale)
        vmax = np.abs(W.bf16_decode(vb[b, l, h])).max()
        err = np.abs(ob[b, l, h * g:(h + 1) * g] - ref).max()
        assert err <= 2.0 ** -8 * vmax, f"unit {u}: out error {err:.3e}"
        got = lse[(u * g):(u + 1) * g].reshape(-1)
        np.testing.assert_allclose(got, rlse / math.log(2.0), rtol=4e-7, atol=6e-5)


def _inputs(seed, B, L, hq, hkv, d, n, n_q):
    rng = np.random.default_rng(seed)
    q = W.bf16_bits((rng.standard_normal((B, L, hq, n_q, d)) / math.sqrt(d)).astype(np.float32))
    k = W.bf16_bits(rng.standard_normal((B, L, hkv, n, d)).astype(np.float32))
    v = W.bf16_bits(rng.standard_normal((B, L, hkv, n, d)).astype(np.float32))
    return rng, q, k, v


@pytest.mark.parametrize("case", [
    # seed, B, L, hq, hkv, d, n, n_q, n_vertical, n_slash
    (1, 1, 1, 4, 2, 128, 700, 700, 30, 10),     # full prefill of a ragged sequence
    (2, 1, 2, 2, 1, 64, 1000, 300, 50, 20),     # the last 300 rows, head_dim 64
    (3, 1, 1, 2, 2, 128, 513, 130, 0, 5),       # no vertical columns
    (4, 1, 1, 4, 1, 128, 600, 257, 40, 0),      # no slash beyond the token itself
    (5, 2, 1, 2, 1, 128, 2000, 256, 200, 64),   # far vertical keys and diagonals
    (6, 1, 2, 6, 2, 128, 800, 300, 40, 12),     # g = 3: the second pair has one head
    (7, 1, 1, 4, 2, 128, 65536, 200, 4096, 100),  # the largest pattern: n = 65536, 4096 vertical keys
])
def test_vs_attention_parity(P, case):
    seed, B, L, hq, hkv, d, n, n_q, n_v, n_s = case
    rng, qb, kb, vb = _inputs(seed, B, L, hq, hkv, d, n, n_q)
    vert, sl = _pattern(rng, B * L * hkv, n, n_v, n_s)
    _check(P, qb, kb, vb, vert, sl, scale=0.9)


def test_vs_attention_full_pattern_is_dense(P):
    # every key vertical: dense causal attention, also against the oracle's prefill attention
    rng, qb, kb, vb = _inputs(7, 1, 1, 2, 1, 128, 300, 300)
    vert = np.arange(300, dtype=np.int32)[None]
    sl = np.zeros((1, 0), np.int32)
    _check(P, qb, kb, vb, vert, sl)
    out, _ = _run(P, qb, kb, vb, vert, sl)
    ref, _ = oracle.prefill_unit(qb[0, 0], kb[0, 0, 0], vb[0, 0, 0], 300, 0, 300)
    assert np.abs(W.bf16_decode(bits_of(out))[0, 0] - ref).max() <= 2.0 ** -8 * np.abs(W.bf16_decode(vb)).max()


def test_vs_attention_deterministic_and_bad_indices(P):
    import torch
    rng, qb, kb, vb = _inputs(8, 1, 1, 4, 2, 128, 900, 400)
    vert, sl = _pattern(rng, 2, 900, 60, 30)
    a, la = _run(P, qb, kb, vb, vert, sl)
    b, lb = _run(P, qb, kb, vb, vert, sl)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)
    assert P.spk_device_error() == (0, 0)
    bad = vert.copy()
    bad[1, -1] = 900                     # outside [0, n): recorded, ignored, nothing faults
    _run(P, qb, kb, vb, bad, sl)
    st, _ = P.spk_device_error()
    assert st == P.binding.SPK_ERR_ARG
    assert P.spk_device_error() == (0, 0)
