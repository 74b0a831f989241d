"""Host-side logic of bench.py, on the CPU: the clock record's summary (median SM clock
under load, throttle reasons), the lookup of recorded DRAM traffic (dropped once the
kernel's source changes), the peak denominators and the unit scaling."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _sampler_with(tmp_path, rows):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        for r in rows:
            f.write(", ".join(str(v) for v in r) + "\n")
    s.proc = object()               # a sampler that ran (summary() only reads the file)
    return s


def test_clock_summary_median_under_load_and_reasons(tmp_path):
    # index, sm MHz, max MHz, power W, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    idle = [(0, 345, 1965, 140.0, "0x1", "Not Active", "Not Active", "Not Active", "Not Active")]
    busy = [(0, mhz, 1965, 900.0, "0x0", "Not Active", "Not Active", "Not Active", cap)
            for mhz, cap in [(1965, "Not Active"), (1950, "Not Active"), (1800, "Active"), (1965, "Not Active")]]
    s = _sampler_with(tmp_path, idle * 3 + busy)
    got = s.summary()
    # idle samples (below half the peak power) are left out of the median and the reasons
    assert got["sm_mhz"] == 1957.5 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    assert got["samples"] == 7 and got["samples_under_load"] == 4


def test_clock_summary_reports_hardware_slowdown(tmp_path):
    rows = [(0, 1200, 1965, 950.0, "0x8", "Active", "Not Active", "Not Active", "Not Active")] * 3
    assert _sampler_with(tmp_path, rows).summary()["reasons"] == ["hw_slowdown"]


def test_clock_summary_without_samples(tmp_path):
    s = _sampler_with(tmp_path, [])
    assert s.summary()["reasons"] == ["no samples"]
    s.proc = None
    assert s.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_recorded_traffic_follows_the_source_sha(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    key, e = next((k, v) for k, v in entries.items() if "@" in k and isinstance(v, dict))
    kernel, workload = key.split("@", 1)
    real = bench.file_sha
    monkeypatch.setattr(bench, "file_sha", lambda path: e["source_sha"])
    assert bench.recorded_traffic(kernel, workload) == e["bytes_per_launch"]
    monkeypatch.setattr(bench, "file_sha", lambda path: "0" * 16)
    assert bench.recorded_traffic(kernel, workload) is None
    monkeypatch.setattr(bench, "file_sha", real)
    assert bench.recorded_traffic(kernel, "no-such-workload") is None


def test_every_traffic_entry_names_a_source_and_a_capture():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    for key, e in entries.items():
        if "@" not in key:
            continue
        assert os.path.exists(os.path.join(ROOT, e["source"])), key
        assert e["bytes_per_launch"] > 0 and "--clock-control none" in e["capture"], key


def test_peaks_and_units():
    peaks, kind = bench.load_peaks()
    assert kind == ("measured" if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else "fallback")
    assert peaks["hbm_gbs"] > 0 and peaks["bf16_tflops"] > 0
    assert bench.scale(2.5e15, "TFLOP/s") == pytest.approx(2500.0)
    assert bench.scale(6.5e12, "GB/s") == pytest.approx(6500.0)
