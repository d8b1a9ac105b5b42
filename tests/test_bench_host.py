"""Host-side logic of bench.py on CPU: the clock record, the committed-traffic
lookup and the peak denominators (no GPU)."""
import json
import os

import bench


def _row(sm, power, *active):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in active else "Not Active" for n in names]
    return ["0", str(sm), "1965", str(power), "0x0"] + flags


def test_clock_summary_uses_loaded_samples_and_reports_active_reasons():
    rows = [_row(1965, 120.0), _row(1650, 990.0, "sw_power_cap"), _row(1700, 995.0, "sw_power_cap"),
            _row(1600, 985.0), ["0", "[N/A]", "1965", "x", "", "", "", "", ""]]
    s = bench.ClockSampler.summarize(rows)
    assert s["sm_mhz"] == 1650.0              # median of the three samples above 300 W
    assert s["power_w"] == 990.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]   # the idle sample's flags are not counted
    assert s["samples"] == 5


def test_clock_summary_of_a_short_run_falls_back_to_every_sample():
    s = bench.ClockSampler.summarize([_row(1900, 150.0), _row(1965, 200.0)])
    assert s["sm_mhz"] == 1932.5 and s["power_w"] is None and s["reasons"] == []


def test_profiled_traffic_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"source_hash": bench.source_hash(["k.cuh"]), "bytes_per_launch": 123.0}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"fwd": rec}))
    assert bench.profiled_traffic("fwd", ["k.cuh"])["bytes_per_launch"] == 123.0
    assert bench.profiled_traffic("mask", ["k.cuh"]) is None
    src.write_text("kernel v2\n")             # the kernel changed since the capture
    assert bench.profiled_traffic("fwd", ["k.cuh"]) is None


def test_measured_peaks_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    fb = bench.measured_peaks()
    assert fb["source"] == "fallback" and fb["bf16_tflops"] > fb["bf16_tflops_sustained"] > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}))
    m = bench.measured_peaks()
    assert m == {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
                 "source": "measured"}


def test_committed_peaks_file_is_readable():
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = bench.measured_peaks()
        assert m["source"] == "measured" and m["bf16_tflops_sustained"] <= m["bf16_tflops"]
