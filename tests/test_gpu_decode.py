"""Decode attention over a compacted cache, through the C ABI, against the
fp64 oracle: ragged row counts, both head sizes, GQA groups up to 8, the
cache that speckv_compress leaves, and bitwise reproducibility.

Tolerance: logits are bf16 products summed in fp32 on the tensor cores and
exponentiated with ex2.approx (relative error ~2^-22); the weights enter the
value product as two bf16 terms (16 significant bits: relative error
<= 2^-17 each) and the sums run in fp32, so the error is ~1e-5 of max|v|;
the bound is 1e-4."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.spk_device_error(clear=True)
    return P


def _check(gpu, ref, vmax):
    np.testing.assert_allclose(gpu, ref, rtol=0, atol=1e-4 * max(vmax, 1e-30))


@pytest.mark.parametrize("case", [
    # seed, B, L, hq, hkv, d, n_kv, scale
    (1, 1, 1, 5, 1, 128, 1, 1.0),          # a single row
    (2, 1, 2, 40, 8, 128, 320, 0.0884),    # Qwen-like group, C_max 256 + window 64
    (3, 2, 1, 32, 8, 128, 1087, 0.125),    # ragged row count (not a multiple of 32)
    (4, 1, 3, 14, 2, 64, 2048, 0.125),     # g = 7, head_dim 64
    (5, 1, 1, 8, 1, 64, 33, 2.0),          # g = 8 (the largest), peaked softmax
    (6, 1, 1, 3, 3, 128, 5, 0.5),          # g = 1, fewer rows than warps
    (7, 1, 2, 16, 4, 128, 385, 0.1),       # 13 blocks: two slots per warp, uneven blocks per warp
    (8, 1, 1, 6, 1, 64, 4097, 0.125),      # long cache at head_dim 64
])
def test_decode_parity(P, case):
    import torch
    seed, B, L, hq, hkv, d, n_kv, scale = case
    rng = np.random.default_rng(seed)
    qb = W.bf16_bits(rng.standard_normal((B, L, hq, d)).astype(np.float32))
    kb = W.bf16_bits(rng.standard_normal((B, L, hkv, n_kv, d)).astype(np.float32))
    vb = W.bf16_bits(rng.standard_normal((B, L, hkv, n_kv, d)).astype(np.float32))
    out = P.decode_attention(to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb), scale=scale)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    ref = oracle.decode_attention(qb, kb, vb, scale)
    _check(out.cpu().numpy(), ref, float(np.abs(W.bf16_decode(vb)).max()))


def test_decode_on_the_compacted_cache(P):
    # score + select + compact, then decode one new token per head over the
    # kept rows: equal to the oracle's decode over the oracle's gathered rows
    import torch
    rng = np.random.default_rng(9)
    B, L, hq, hkv, d, n_in, nw, nl, c_max = 1, 2, 8, 2, 128, 1500, 32, 32, 128
    R = nw + nl
    qb = W.bf16_bits((rng.standard_normal((B, L, hq, R, d)) / np.sqrt(d)).astype(np.float32))
    kb = W.bf16_bits(rng.standard_normal((B, L, hkv, n_in, d)).astype(np.float32))
    vb = W.bf16_bits(rng.standard_normal((B, L, hkv, n_in, d)).astype(np.float32))
    buf = P.speckv_compress(to_bf16_tensor(qb), to_bf16_tensor(kb), to_bf16_tensor(vb), nw, c_max, 7)
    qd = W.bf16_bits(rng.standard_normal((B, L, hq, d)).astype(np.float32))
    out = P.decode_attention(to_bf16_tensor(qd), buf.k_out, buf.v_out, scale=d ** -0.5)
    torch.cuda.synchronize()
    idx = buf.idx.cpu().numpy().reshape(B, L, hkv, -1)
    kc = np.take_along_axis(kb, idx[..., None], axis=3)
    vc = np.take_along_axis(vb, idx[..., None], axis=3)
    ref = oracle.decode_attention(qd, kc, vc, d ** -0.5)
    _check(out.cpu().numpy(), ref, float(np.abs(W.bf16_decode(vc)).max()))


def test_decode_is_deterministic(P):
    import torch
    rng = np.random.default_rng(10)
    q = to_bf16_tensor(W.bf16_bits(rng.standard_normal((1, 4, 40, 128)).astype(np.float32)))
    k = to_bf16_tensor(W.bf16_bits(rng.standard_normal((1, 4, 8, 700, 128)).astype(np.float32)))
    v = to_bf16_tensor(W.bf16_bits(rng.standard_normal((1, 4, 8, 700, 128)).astype(np.float32)))
    a = P.decode_attention(q, k, v, scale=0.09)
    b = P.decode_attention(q, k, v, scale=0.09)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
