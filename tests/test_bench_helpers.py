"""Host-side bookkeeping of bench.py (no GPU): the roofline denominators, the
DRAM-traffic gate and the exponential-stream peak."""
import json

import bench


def test_tensor_peak_is_the_burst_figure():
    # kernels are timed per launch (milliseconds), so the burst GEMM figure
    # is the denominator; the sustained one is context only
    peak, src = bench.tensor_peak({"bf16_tflops": 1615.5, "bf16_tflops_sustained": 1379.5, "source": "measured"})
    assert peak == 1615.5 and "burst" in src
    r = bench.kernel_roofline("k", 10.0, 8.0e12, {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
                                                 "hbm_gbs": 6500.0, "source": "measured"})
    assert abs(r["achieved"] - 800.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12
    assert abs(r["frac_of_sustained"] - 800.0 / 1400.0) < 1e-12


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    digests = {k: bench.kernel_source_digest(k) for k in bench.KERNEL_SOURCES}
    rec = {"kernels": {"score_colsum_pass": {"source_sha256": digests["score_colsum_pass"], "workloads": {"w": 123}},
                       "vs_attn_kernel": {"source_sha256": "0" * 64, "workloads": {"w": 7}}}}
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digests read the kernel sources from ROOT too: point them back at the repository's
    monkeypatch.setattr(bench, "kernel_source_digest", lambda k="score_colsum_pass": digests[k])
    assert bench.captured_traffic("score_colsum_pass", "w") == 123
    assert bench.captured_traffic("score_colsum_pass", "other") is None
    assert bench.captured_traffic("score_lse_pass", "w") is None        # not captured
    assert bench.captured_traffic("vs_attn_kernel", "w") is None        # captured from other sources
    rec["kernels"]["score_colsum_pass"]["source_sha256"] = "0" * 64
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.captured_traffic("score_colsum_pass", "w") is None


def test_digests_cover_each_kernels_sources():
    a = bench.kernel_source_digest()
    assert len(a) == 64 and a == bench.kernel_source_digest("score_colsum_pass")
    assert "decode.cu" not in bench.SCORING_SOURCES and "score.cu" in bench.SCORING_SOURCES
    assert "api.cu" not in bench.SCORING_SOURCES
    assert "attn.cu" in bench.KERNEL_SOURCES["prefill_attention"] and "vs.cu" in bench.KERNEL_SOURCES["vs_attn_kernel"]
    assert len({bench.kernel_source_digest(k) for k in ("score_lse_pass", "prefill_attention", "vs_attn_kernel")}) == 3


def test_exp2_peak_from_unit_counts():
    # 148 SMs x (16 MUFU / (1 - 0.4 polynomial share)) per clock x 1965 MHz
    assert abs(bench.exp2_peak_per_s() - 148 * 16 / 0.6 * 1965e6) < 1.0


def test_suite_names_resolve():
    for name in bench.SUITE:
        cfg = bench.config_of(name)
        assert cfg is not None
    assert bench.config_of("qwen2.5-32b_speckv_64k@2048").c_max == 2048
    assert bench.config_of("qwen2.5-32b_speckv_64k+prefill", layers=2).layers == 2


def test_vs_tile_count_matches_a_direct_walk():
    # the bench's count of processed key tiles equals a plain per-tile check
    # of "some offset of S u {0} hits the tile" plus the vertical tiles
    import dataclasses
    import numpy as np
    import workloads as W
    cfg = dataclasses.replace(W.VS_LLAMA8B_16K, layers=1, hkv=2, hq=4, n=1000, n_q=700, n_vertical=50,
                              n_local=8, n_far=5)
    vert, sl = W.vs_pattern(cfg, seed=3)
    tiles, _ = bench.vs_tile_work(cfg, vert, sl)
    ref = 0
    for u in range(cfg.units):
        S = set(sl[u].tolist()) | {0}
        V = vert[u].numpy()
        for rb in range((cfg.n_q + 127) // 128):
            p0 = cfg.n - cfg.n_q + rb * 128
            pl = cfg.n - cfg.n_q + min(rb * 128 + 127, cfg.n_q - 1)
            for t in range(pl // 128 + 1):
                if any(p0 - 128 * t - 127 <= o <= pl - 128 * t for o in S):
                    ref += 1
            ref += (int((V <= pl).sum()) + 127) // 128
    assert tiles == ref * cfg.g


def test_cpu_baselines_on_tiny_workloads():
    # the oracle-timing plumbing: spawned processes draw their own inputs and
    # report oracle seconds; the value is the timed work over (CPU-s / cores)
    import dataclasses
    import workloads as W
    full = bench.cpu_baseline_speckv(W.TINY, 0, 2, full=True)
    assert full["kind"] == "oracle" and full["cores"] == 2 and full["value"] > 0
    cfg = dataclasses.replace(W.TINY, layers=2)
    part = bench.cpu_baseline_speckv(cfg, 0, 2)
    assert part["value"] > 0 and "1 of its 2 query heads" in part["sample"]
    pc = W.SpecPCConfig("tiny_pc", batch=1, layers=3, l_skip=1, hq=4, hkv=2, head_dim=64, n_in=300,
                        n_rows=32, n_lookahead=1, keep=40)
    r = bench.cpu_baseline_specpc(pc, 0, 2)
    assert r["value"] > 0 and "2 (batch, layer)" in r["sample"]
    cc = W.CascadeConfig("tiny_cascade", draft=dataclasses.replace(pc, batch=2, keep=96),
                         target=W.SpecKVConfig("t", batch=2, layers=1, hq=4, hkv=2, head_dim=64, n_in=96,
                                               n_window=8, n_lookahead=8, c_max=16),
                         n_in_full=300)
    r = bench.cpu_baseline_cascade(cc, 0, 2)
    assert r["value"] > 0 and "extrapolated" in r["sample"]
