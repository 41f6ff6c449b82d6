"""Host logic of bench.py on CPU: the clock record that decides whether a timed
run is valid, and the guard that reports the ncu traffic figure only for the
kernel sources it was taken on."""
import os

import bench


def _csv(tmp_path, rows):
    p = os.path.join(str(tmp_path), "clocks.csv")
    with open(p, "w") as f:
        for r in rows:
            f.write(", ".join(str(x) for x in r) + "\n")
    return p


def test_clock_record_without_throttling(tmp_path):
    rows = [(0, mhz, 1965, 250.0, "0x0000000000000000", "Not Active", "Not Active", "Not Active", "Not Active")
            for mhz in (1965, 1965, 1950)]
    got = bench.ClockSampler.parse(_csv(tmp_path, rows))
    assert got == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}


def test_clock_record_reports_active_reasons(tmp_path):
    rows = [(0, 1965, 1965, 700.0, "0x0", "Not Active", "Not Active", "Not Active", "Active"),
            (0, 1500, 1965, 990.0, "0x0", "Active", "Not Active", "Not Active", "Active"),
            (0, "[N/A]", 1965, 0.0, "0x0", "Not Active", "Not Active", "Active", "Not Active"),  # unparsable clock
            ("garbage line",)]
    got = bench.ClockSampler.parse(_csv(tmp_path, rows))
    assert got["samples"] == 2 and got["sm_mhz"] == 1732.5
    assert got["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_record_empty(tmp_path):
    assert bench.ClockSampler.parse(_csv(tmp_path, [])) is None


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    wl = "qwen2.5-omni-3b-36L-b1-ctx10240"
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURE", {"sources_sha256": bench.kernel_sources_sha256(),
                                                   "bytes_per_launch": 123})
    assert bench.captured_traffic(wl) == 123
    assert bench.captured_traffic("qwen2.5-omni-3b-36L-b16-ctx32768") is None  # another workload
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURE", {"sources_sha256": "0" * 64, "bytes_per_launch": 123})
    assert bench.captured_traffic(wl) is None                                  # sources changed since
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURE", {"sources_sha256": None, "bytes_per_launch": None})
    assert bench.captured_traffic(wl) is None


def test_peak_source():
    peak, kind = bench.peaks()
    assert peak > 0 and kind in ("measured", "fallback")
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured"
