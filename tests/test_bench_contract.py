"""Host-side pieces of bench.py's report: the DRAM traffic of the roofline
comes from the committed ncu capture only while the GEMM source is the one
the capture was taken on, and the peaks come from the measured file when
present."""

import json

import bench


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "sparse_mixture_experts_06_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "gemm_sm100.cu").write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.gemm_source_hash()
    rec = {"up_swiglu_gemm": {"source_sha256_16": h, "bytes_per_launch": 123}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_record("up_swiglu_gemm")["bytes_per_launch"] == 123
    assert bench.traffic_record("down_combine_gemm") is None
    (src / "gemm_sm100.cu").write_text("// kernel v2\n")  # the kernel changed since the capture
    assert bench.traffic_record("up_swiglu_gemm") is None


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk, kind = bench.peaks()
    assert kind == "fallback" and pk["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    pk, kind = bench.peaks()
    assert kind == "measured" and pk["bf16_tflops"] == 2.0
