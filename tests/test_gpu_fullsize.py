"""Parity at the full workload sizes, in the launch configuration bench.py
times (SpeckvBuffers + speckv_compress over every unit).

The oracle runs on sampled units (first, middle, last); every unit is checked
through properties that hold at any size: prefix + window attention mass =
g * R, indices ascending and unique with the window appended, compacted K/V
equal to K/V at the indices bit for bit, and the selection equal to the
oracle's pool + top-k applied to the GPU's own scores.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import assert_indices_match, assert_scores_close, bits_of

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def P():
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.spk_device_error(clear=True)
    return P


def _check_speckv_full(P, cfg, sample_units):
    import torch
    from prompt_compression_b200.pipeline import SpeckvBuffers
    inp = W.speckv_inputs(cfg, seed=7, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    buf = SpeckvBuffers(q, k, v, cfg.n_window, cfg.c_max, window_mass=True)
    P.speckv_compress(q, k, v, cfg.n_window, cfg.c_max, cfg.pool, buffers=buf)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    g, R, c = cfg.g, cfg.rows, min(cfg.c_max, cfg.n_pre)

    # ---- every unit: conservation, index structure, compaction (on the device)
    tot = buf.scores.double().sum(1) + buf.window_mass.double().sum(1)
    assert torch.allclose(tot, torch.full_like(tot, g * R), rtol=1e-4, atol=0), tot.min().item()
    idx = buf.idx.long()
    assert bool((idx[:, 1:c] > idx[:, :c - 1]).all())
    assert bool((idx[:, c:] == torch.arange(cfg.n_pre, cfg.n_in, device="cuda")).all())
    kk = k.view(cfg.units, cfg.n_in, cfg.head_dim)
    vv = v.view(cfg.units, cfg.n_in, cfg.head_dim)
    gather = idx[:, :, None].expand(-1, -1, cfg.head_dim)
    assert torch.equal(buf.k_out.view(cfg.units, -1, cfg.head_dim).view(torch.int16),
                       torch.gather(kk, 1, gather).view(torch.int16))
    assert torch.equal(buf.v_out.view(cfg.units, -1, cfg.head_dim).view(torch.int16),
                       torch.gather(vv, 1, gather).view(torch.int16))

    # ---- sampled units against the fp64 oracle
    for u in sample_units:
        b, l, h = u // (cfg.layers * cfg.hkv), (u // cfg.hkv) % cfg.layers, u % cfg.hkv
        qb = bits_of(q[b, l, h * g:(h + 1) * g])
        kb = bits_of(k[b, l, h])
        s, wm = oracle.speckv_unit(qb, kb, cfg.n_window, cfg.n_lookahead)
        gs = buf.scores[u].cpu().numpy()
        assert_scores_close(gs, s, f"{cfg.name} unit {u} scores")
        assert_scores_close(buf.window_mass[u].cpu().numpy(), wm, f"{cfg.name} unit {u} window mass")
        p = oracle.maxpool(s, cfg.pool)
        gi = buf.idx[u].cpu().numpy()
        own = oracle.topk_with_tail(oracle.maxpool(gs.astype(np.float64), cfg.pool), cfg.c_max, cfg.n_window)
        assert np.array_equal(gi, own), f"unit {u}: selection differs from the oracle on the GPU's scores"
        assert_indices_match(gi, oracle.topk_with_tail(p, cfg.c_max, cfg.n_window), p, c)
    return inp, buf


def test_llama8b_16k_full(P):
    cfg = W.LLAMA8B_16K
    _check_speckv_full(P, cfg, [0, cfg.units // 2 + 3, cfg.units - 1])


def test_qwen32b_64k_full(P):
    cfg = W.QWEN32B_64K
    inp, buf = _check_speckv_full(P, cfg, [0, cfg.units - 1])
    # planted heavy keys (1% of the prefix) fill the kept slots far above the
    # 1% a random selection would give; the fraction itself is reported
    heavy = set(inp["heavy"][0].tolist())
    idx = buf.idx.cpu().numpy()[:, :cfg.c_max]
    hits = np.mean([len(heavy & set(r.tolist())) / min(cfg.c_max, len(heavy)) for r in idx])
    print(f"heavy-key share of the kept slots: {hits:.3f}")
    assert hits > 0.1, hits


def test_qwen32b_64k_cmax_sweep(P):
    """C_max in {1024, 2048} on sampled units of the 64K workload."""
    import dataclasses
    import torch
    for c_max in (1024, 2048):
        cfg = dataclasses.replace(W.QWEN32B_64K, layers=2, c_max=c_max)
        _check_speckv_full(P, cfg, [0, cfg.units - 1])
        torch.cuda.empty_cache()


def test_specpc_qwen05b_32k_full(P):
    import torch
    cfg = W.QWEN05B_SPECPC_32K
    inp = W.specpc_inputs(cfg, seed=3, device="cuda")
    w = W.specpc_row_weights(cfg.n_rows).astype(np.float32)
    wt = torch.from_numpy(w).cuda()
    scores, idx = P.specpc_select(inp["q"], inp["k"], wt, cfg.l_skip, cfg.keep, cfg.pool, cfg.n_lookahead)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    ref = oracle.specpc_batch(bits_of(inp["q"][0]), bits_of(inp["k"][0]), w.astype(np.float64), cfg.l_skip,
                              cfg.n_lookahead)
    gs = scores[0].cpu().numpy()
    assert_scores_close(gs, ref, "specpc 32K scores")
    p = oracle.maxpool(ref, cfg.pool)
    gi = idx[0].cpu().numpy()
    assert np.array_equal(gi, oracle.topk_with_tail(oracle.maxpool(gs.astype(np.float64), cfg.pool), cfg.keep, 0))
    assert_indices_match(gi, oracle.topk_with_tail(p, cfg.keep, 0), p, cfg.keep)


def test_cascade_128k_full(P):
    """SpecKV-PC at 128K, batch 2: SpecPC on the draft keeps 2048 tokens, the
    target K/V are gathered there, SpecKV keeps 256 + 64 of them.  Step 2 is
    checked against the oracle on sampled units, the gather bit for bit; the
    SpecPC step at this length is checked at full n_in on a one-layer draft."""
    import torch
    cc = W.CASCADE_128K
    d, t = cc.draft, cc.target
    dr = W.specpc_inputs(d, seed=11, device="cuda")
    heavy = dr["heavy"]
    tcfg_full = W.SpecKVConfig("cascade_target_128k", batch=t.batch, layers=t.layers, hq=t.hq, hkv=t.hkv,
                               head_dim=t.head_dim, n_in=cc.n_in_full, n_window=t.n_window,
                               n_lookahead=t.n_lookahead, c_max=t.c_max, heavy_frac=t.heavy_frac)
    tg = W.speckv_inputs(tcfg_full, seed=12, device="cuda", heavy_pos=heavy)
    w = torch.from_numpy(W.specpc_row_weights(d.n_rows).astype(np.float32)).cuda()
    pc_scores, pc_idx, k_g, v_g, out = P.cascade_compress(dr["q"], dr["k"], w, d.l_skip, d.keep, tg["q"], tg["k"],
                                                          tg["v"], t.n_window, t.c_max)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    pidx = pc_idx.long()
    assert pidx.shape == (d.batch, d.keep)
    assert bool((pidx[:, 1:] > pidx[:, :-1]).all())
    # gather of the target cache at the SpecPC indices, every (layer, KV head)
    for b in range(d.batch):
        gk = tg["k"][b].index_select(2, pidx[b])
        assert torch.equal(k_g[b].view(torch.int16), gk.view(torch.int16))
        assert torch.equal(v_g[b].view(torch.int16), tg["v"][b].index_select(2, pidx[b]).view(torch.int16))
    # step 2 on sampled units
    g = t.g
    kgb = k_g
    for u in (0, t.batch * t.layers * t.hkv - 1):
        b, l, h = u // (t.layers * t.hkv), (u // t.hkv) % t.layers, u % t.hkv
        s, wm = oracle.speckv_unit(bits_of(tg["q"][b, l, h * g:(h + 1) * g]), bits_of(kgb[b, l, h]),
                                   t.n_window, t.n_lookahead)
        assert_scores_close(out.scores[u].cpu().numpy(), s, f"cascade step-2 unit {u}")
        p = oracle.maxpool(s, t.pool)
        assert_indices_match(out.idx[u].cpu().numpy(), oracle.topk_with_tail(p, t.c_max, t.n_window), p,
                             t.c_max)
    del tg, k_g, v_g, out
    torch.cuda.empty_cache()
    # SpecPC parity at n_in = 131072 on a draft with one scored layer
    q1 = dr["q"][:1, d.l_skip - 1:d.l_skip + 1].contiguous()
    k1 = dr["k"][:1, d.l_skip - 1:d.l_skip + 1].contiguous()
    s1, _ = P.specpc_select(q1, k1, w, 1, d.keep, d.pool, d.n_lookahead)
    torch.cuda.synchronize()
    ref = oracle.specpc_batch(bits_of(q1[0]), bits_of(k1[0]), W.specpc_row_weights(d.n_rows).astype(np.float32)
                              .astype(np.float64), 1, d.n_lookahead)
    assert_scores_close(s1[0].cpu().numpy(), ref, "specpc 128K one-layer scores")


def _sample_rows(rng, g, R, extra=8, boundaries=()):
    """(query head, row) pairs to check: the first and last row of every
    query head, the given rows of head 0, and a few random ones."""
    rows = {(h, 0) for h in range(g)} | {(h, R - 1) for h in range(g)}
    rows |= {(0, i) for i in boundaries if 0 <= i < R}
    target = len(rows) + extra
    while len(rows) < target:
        rows.add((int(rng.integers(g)), int(rng.integers(R))))
    return sorted(rows)


def test_prefill_attention_qwen32b_64k_full(P):
    """The prefill attention of the window and lookahead rows at the 64K
    workload, launched as the +prefill step launches it (every unit, the
    column pass's workspace filled), then the column pass on its row offsets.
    Sampled rows of sampled units against the fp64 oracle (output and
    input-key LSE); every unit through properties (each output row is a
    convex combination of V rows, every LSE finite, each row's attention mass
    over the input keys is 1); the scores of a sampled unit against the
    oracle."""
    import torch
    from prompt_compression_b200.pipeline import SpeckvBuffers
    cfg = W.QWEN32B_64K
    inp = W.speckv_inputs(cfg, seed=7, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    gen = torch.Generator(device="cuda").manual_seed(24)
    lshape = (cfg.batch, cfg.layers, cfg.hkv, cfg.n_lookahead, cfg.head_dim)
    k_look = torch.randn(lshape, generator=gen, device="cuda").to(torch.bfloat16)
    v_look = torch.randn(lshape, generator=gen, device="cuda").to(torch.bfloat16)
    buf = SpeckvBuffers(q, k, v, cfg.n_window, cfg.c_max, window_mass=True)
    g, R, nw, nl, n_in, d = cfg.g, cfg.rows, cfg.n_window, cfg.n_lookahead, cfg.n_in, cfg.head_dim
    lse2 = torch.empty((cfg.units, g * R), dtype=torch.float32, device="cuda")
    out = P.speckv_prefill_attention(q, k, v, k_look, v_look, nw, lse2=lse2, workspace=buf.ws_score)
    P.speckv_colsum(q, k, nw, buf.scores, buf.ws_score, window_mass=buf.window_mass)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)

    # ---- every unit
    assert bool(torch.isfinite(lse2).all())
    vmax = torch.maximum(v.view(cfg.units, -1).abs().amax(1), v_look.view(cfg.units, -1).abs().amax(1)).float()
    omax = out.view(cfg.units, -1).abs().amax(1).float()
    assert bool((omax <= vmax * (1 + 2.0 ** -8)).all()), (omax - vmax).max().item()
    tot = buf.scores.double().sum(1) + buf.window_mass.double().sum(1)
    assert torch.allclose(tot, torch.full_like(tot, g * R), rtol=1e-4, atol=0), tot.min().item()

    # ---- sampled rows of sampled units against the oracle
    rng = np.random.default_rng(1)
    for u in (0, cfg.units - 1):
        b, l, h = u // (cfg.layers * cfg.hkv), (u // cfg.hkv) % cfg.layers, u % cfg.hkv
        qb = bits_of(q[b, l, h * g:(h + 1) * g])
        kb = np.concatenate([bits_of(k[b, l, h]), bits_of(k_look[b, l, h])])
        vb = np.concatenate([bits_of(v[b, l, h]), bits_of(v_look[b, l, h])])
        rows = _sample_rows(rng, g, R, boundaries=(nw - 1, nw, 127, 128))
        ref, rlse = oracle.prefill_unit(qb, kb, vb, nw, nl, n_in, rows=rows)
        ob = W.bf16_decode(bits_of(out[b, l, h * g:(h + 1) * g])).astype(np.float64)
        got = np.stack([ob[hh, i] for hh, i in rows])
        bound = 2.0 ** -8 * np.abs(W.bf16_decode(vb)).max()
        err = np.abs(got - ref).max()
        assert err <= bound, f"unit {u}: out error {err:.3e} > {bound:.3e}"
        lg = lse2[u].cpu().numpy()
        np.testing.assert_allclose([lg[hh * R + i] for hh, i in rows], rlse / math.log(2.0), rtol=4e-7, atol=6e-5)
    u = cfg.units - 1
    b, l, h = u // (cfg.layers * cfg.hkv), (u // cfg.hkv) % cfg.layers, u % cfg.hkv
    s, wm = oracle.speckv_unit(bits_of(q[b, l, h * g:(h + 1) * g]), bits_of(k[b, l, h]), nw, nl)
    assert_scores_close(buf.scores[u].cpu().numpy(), s, f"scores from the prefill's row offsets, unit {u}")
    assert_scores_close(buf.window_mass[u].cpu().numpy(), wm, f"window mass from the prefill, unit {u}")
    del inp, q, k, v, k_look, v_look, buf, out
    torch.cuda.empty_cache()


def test_decode_qwen32b_compressed_full(P):
    """Decode over the compressed cache at the benched shape (64 layers x 40
    query heads over 320 kept rows per KV head): every output against the
    oracle; then over the full 65,536-row cache, sampled layers against the
    oracle (tolerance as in the decode parity tests: 1e-4 of max |v|)."""
    import torch
    cfg = W.DECODE_QWEN32B
    B_, L, hq, hkv, d = cfg.batch, cfg.layers, cfg.hq, cfg.hkv, cfg.head_dim
    gen = torch.Generator(device="cuda").manual_seed(5)

    def rnd(*shape):
        return torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16)

    scale = d ** -0.5
    q = rnd(B_, L, hq, d)
    kc, vc = rnd(B_, L, hkv, cfg.n_kv, d), rnd(B_, L, hkv, cfg.n_kv, d)
    out = torch.empty((B_, L, hq, d), dtype=torch.float32, device="cuda")
    P.decode_attention(q, kc, vc, out, scale)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    ref = oracle.decode_attention(bits_of(q), bits_of(kc), bits_of(vc), scale)
    vmax = float(vc.abs().max())
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=1e-4 * vmax)

    kf, vf = rnd(B_, L, hkv, cfg.n_kv_full, d), rnd(B_, L, hkv, cfg.n_kv_full, d)
    P.decode_attention(q, kf, vf, out, scale)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)
    for l in (0, L - 1):
        ref = oracle.decode_attention(bits_of(q[:, l:l + 1]), bits_of(kf[:, l:l + 1]), bits_of(vf[:, l:l + 1]),
                                      scale)
        vmax = float(vf[:, l].abs().max())
        np.testing.assert_allclose(out[:, l:l + 1].cpu().numpy(), ref, rtol=0, atol=1e-4 * vmax)
    del kf, vf
    torch.cuda.empty_cache()


def test_vs_llama8b_16k_full(P):
    """Vertical-Slash sparse prefill at the benched workload (32 layers, every
    one of the 16,384 rows, 1024 vertical keys and 80 diagonals per unit):
    sampled rows of sampled units against the fp64 oracle (output within
    2^-8 of max |v|, LSE as in the Vertical-Slash parity tests), every unit
    through properties (outputs convex combinations of V rows, LSE finite)."""
    import torch
    cfg = W.VS_LLAMA8B_16K
    gen = torch.Generator(device="cuda").manual_seed(9)
    shape_q = (cfg.batch, cfg.layers, cfg.hq, cfg.n_q, cfg.head_dim)
    shape_k = (cfg.batch, cfg.layers, cfg.hkv, cfg.n, cfg.head_dim)
    q = (torch.randn(shape_q, generator=gen, device="cuda") / cfg.head_dim ** 0.5).to(torch.bfloat16)
    k = torch.randn(shape_k, generator=gen, device="cuda").to(torch.bfloat16)
    v = torch.randn(shape_k, generator=gen, device="cuda").to(torch.bfloat16)
    vert, sl = W.vs_pattern(cfg, seed=9, device="cuda")
    ws = torch.empty(P.vs_workspace_size(P.binding.vs_shape(q, k, cfg.n_vertical, cfg.n_slash)), dtype=torch.uint8,
                     device="cuda")
    lse2 = torch.empty((cfg.batch * cfg.layers * cfg.hq, cfg.n_q), dtype=torch.float32, device="cuda")
    out = P.vs_sparse_attention(q, k, v, vert, sl, lse2=lse2, workspace=ws)
    torch.cuda.synchronize()
    assert P.spk_device_error() == (0, 0)

    g = cfg.g
    assert bool(torch.isfinite(lse2).all())
    vmax = v.view(cfg.units, -1).abs().amax(1).float()
    omax = out.view(cfg.units, -1).abs().amax(1).float()
    assert bool((omax <= vmax * (1 + 2.0 ** -8)).all()), (omax - vmax).max().item()

    rng = np.random.default_rng(2)
    vert_c, sl_c = vert.cpu().numpy(), sl.cpu().numpy()
    for u in (0, cfg.units // 2 + 1, cfg.units - 1):
        b, l, h = u // (cfg.layers * cfg.hkv), (u // cfg.hkv) % cfg.layers, u % cfg.hkv
        qb = bits_of(q[b, l, h * g:(h + 1) * g])
        kb, vb = bits_of(k[b, l, h]), bits_of(v[b, l, h])
        rows = _sample_rows(rng, g, cfg.n_q, extra=12, boundaries=(1, 127, 128, 8191, 8192))
        ref, rlse = oracle.vs_attention_unit(qb, kb, vb, vert_c[u], sl_c[u], rows=rows)
        ob = W.bf16_decode(bits_of(out[b, l, h * g:(h + 1) * g])).astype(np.float64)
        got = np.stack([ob[hh, i] for hh, i in rows])
        bound = 2.0 ** -8 * np.abs(W.bf16_decode(vb)).max()
        err = np.abs(got - ref).max()
        assert err <= bound, f"unit {u}: out error {err:.3e} > {bound:.3e}"
        lg = lse2[u * g:(u + 1) * g].cpu().numpy()
        np.testing.assert_allclose([lg[hh, i] for hh, i in rows], rlse / math.log(2.0), rtol=4e-7, atol=6e-5)
    del q, k, v, out, lse2, ws
    torch.cuda.empty_cache()
