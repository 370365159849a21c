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


class _FakeNvml:
    """Read-only NVML stand-in: two GPUs, the second one the benchmarked one,
    its clock held at 1500 MHz by the power cap."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    class _Pci:
        def __init__(self, bid):
            self.busId = bid

    def nvmlInit(self):
        pass

    def nvmlDeviceGetCount(self):
        return 2

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetPciInfo(self, h):
        return self._Pci([b"00000000:1A:00.0", b"00000000:1B:00.0"][h])

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert h == 1 and kind == self.NVML_CLOCK_SM
        return 1500

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.nvmlClocksEventReasonSwPowerCap | 0x1  # 0x1 (idle) is not a reason the report keeps

    def nvmlDeviceGetPowerUsage(self, h):
        return 998000  # mW


def test_clock_sampler_reads_the_benchmarked_gpu_through_nvml(monkeypatch):
    import sys
    import time
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml())
    s = bench.ClockSampler("0000:1b:00")
    s.start()
    time.sleep(0.05)
    c = s.stop()
    assert c["samples"] >= 2 and c["sm_mhz"] == 1500.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 998.0
    assert "NVML" in c["source"]


def test_roofline_peak_follows_the_sampled_clock_regime():
    """The up GEMM's roofline is held to the sustained bf16 figure when the
    clock sampled during the timed steps was held well below its maximum (the
    power cap over a long run), to the burst figure at full clock or when no
    clock was sampled."""
    import bench
    assert bench.clock_regime(None) == "burst"
    assert bench.clock_regime({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}) == "burst"
    assert bench.clock_regime({"sm_mhz": 1850.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}) == "burst"
    assert bench.clock_regime({"sm_mhz": 1455.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}) == "sustained"
    assert bench.clock_regime({"sm_mhz": None, "sm_max_mhz": 1965.0}) == "burst"
