"""Host-side bookkeeping of bench.py (no GPU): the roofline denominators, the
DRAM-traffic gate and the exponential-stream peak."""
import json

import bench


def test_tensor_peak_prefers_the_sustained_figure():
    peak, src = bench.tensor_peak({"bf16_tflops": 1615.5, "bf16_tflops_sustained": 1379.5, "source": "measured"})
    assert peak == 1379.5 and "sustained" in src
    peak, src = bench.tensor_peak({"bf16_tflops": 1615.5, "bf16_tflops_sustained": None, "source": "measured"})
    assert peak == 1615.5 and "burst" in src


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    digest = bench.kernel_source_digest()
    rec = {"source_sha256": digest, "score_colsum_pass": {"w": 123}}
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digest reads the kernel sources from ROOT too: point it back at the repository's
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    assert bench.captured_traffic("score_colsum_pass", "w") == 123
    assert bench.captured_traffic("score_lse_pass", "w") is None
    rec["source_sha256"] = "0" * 64
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.captured_traffic("score_colsum_pass", "w") is None


def test_digest_covers_the_scoring_sources_only():
    a = bench.kernel_source_digest()
    assert len(a) == 64 and a == bench.kernel_source_digest()
    assert "decode.cu" not in bench.SCORING_SOURCES and "score.cu" in bench.SCORING_SOURCES


def test_exp2_peak_from_unit_counts():
    # 148 SMs x (16 MUFU / (1 - 0.4 polynomial share)) per clock x 1965 MHz
    assert abs(bench.exp2_peak_per_s() - 148 * 16 / 0.6 * 1965e6) < 1.0
