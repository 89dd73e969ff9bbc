"""Host logic of bench.py that needs no GPU: the clock-sample summary the JSON line carries, and the
roofline denominators' source (the measured peaks file, else the stated fallback)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _summary_of(tmp_path, lines, index=0):
    cs = bench.ClockSampler(index)
    cs.out = open(os.path.join(tmp_path, "clocks.csv"), "w+")
    cs.out.write("".join(line + "\n" for line in lines))
    cs.proc = object()   # a sampler that ran
    return cs.summary()


def test_clock_summary_median_max_and_active_reasons(tmp_path):
    na, act = "Not Active", "Active"
    rows = [f"0, {mhz}, 1965, 900.0, 0x0, {na}, {na}, {na}, {pc}"
            for mhz, pc in ((1965, na), (1950, act), (1900, act), (1965, na), (1920, na))]
    s = _summary_of(tmp_path, rows)
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 5


def test_clock_summary_keeps_only_its_gpu_and_reports_throttling(tmp_path):
    na, act = "Not Active", "Active"
    rows = [f"0, 1965, 1965, 900.0, 0x0, {na}, {na}, {na}, {na}",
            f"1, 1200, 1965, 500.0, 0x0, {act}, {act}, {na}, {na}",   # another GPU's samples
            f"0, 1800, 1965, 900.0, 0x0, {na}, {na}, {act}, {na}"]
    s = _summary_of(tmp_path, rows, index=0)
    assert s["samples"] == 2 and s["sm_mhz"] == (1965.0 + 1800.0) / 2
    assert s["reasons"] == ["sw_thermal_slowdown"]
    assert _summary_of(tmp_path, [], index=0)["reasons"] == ["no samples"]


def test_clock_summary_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    assert cs.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.PEAKS_FALLBACK
    with open(os.path.join(tmp_path, "MEASURED_PEAKS.json"), "w") as f:
        json.dump({"hbm_gbs": 6458.1, "bf16_tflops": 1672.0}, f)
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["hbm_gbs"] == 6458.1


def test_routing_stats_of_a_count_vector():
    # T = 8 tokens, k = 2: 16 routed slots over E = 4 experts
    st = bench.routing_stats([8, 4, 4, 0], 8, 2)
    assert st == {"rows_max": 8, "rows_min": 0, "rows_mean": 4.0, "rows_variance": 8.0, "idle_experts": 1,
                  "max_vio": 1.0}
    assert bench.routing_stats([4, 4, 4, 4], 8, 2)["max_vio"] == 0.0   # perfectly balanced
