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
    wl = "qwen3-omni-30b-48L-b8-ctx65536"
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURES", {(wl, "fp16"): {"sources_sha256": bench.kernel_sources_sha256(),
                                                                   "bytes_per_launch": 123}})
    assert bench.captured_traffic(wl) == 123
    assert bench.captured_traffic(wl, "mx") is None                            # another metadata format
    assert bench.captured_traffic("qwen2.5-omni-3b-36L-b16-ctx32768") is None  # another workload
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURES", {(wl, "fp16"): {"sources_sha256": "0" * 64,
                                                                   "bytes_per_launch": 123}})
    assert bench.captured_traffic(wl) is None                                  # sources changed since


def test_kernel_sources_cover_the_decode_sources():
    """Every kernel source the decode and step kernels include is hashed (the
    public header outside the source folder holds declarations only)."""
    import os
    import re
    d = os.path.join(os.path.dirname(bench.__file__), "bit_kv_cache_pack_b200", "csrc")
    seen, todo = set(), ["decode_split_k.cu"]
    while todo:
        name = todo.pop()
        if name in seen or "/" in name or not os.path.exists(os.path.join(d, name)):
            continue
        seen.add(name)
        with open(os.path.join(d, name)) as f:
            todo += re.findall(r'#include "([^"]+)"', f.read())
    assert seen <= set(bench.KERNEL_SOURCES), sorted(seen - set(bench.KERNEL_SOURCES))


def test_both_arms_share_the_config_object():
    """The GPU arm and the oracle arm print the same `config` dict, and the
    default workload is the largest single-GPU configuration (48 layers, 8 x
    65,536 tokens)."""
    import sys
    from synth.workloads import WORKLOADS
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        default = bench.parse_args().workload
    finally:
        sys.argv = argv
    spec = WORKLOADS[default]
    cfg = bench.workload_config(spec, 1)
    assert cfg["workload"] == "qwen3-omni-30b-48L-b8-ctx65536"
    assert cfg["layers"] == 48 and cfg["global_batch"] == 8 and cfg["context"] == 65536
    assert bench.workload_config(spec, 1) == cfg


def test_oracle_sample_is_bounded():
    """The timed oracle sample of the big workloads is one layer of at most four
    sequences; small workloads are timed (nearly) whole."""
    from synth.workloads import WORKLOADS
    assert bench.oracle_sample_shape(WORKLOADS["omni30b-b8"]) == (1, 4)
    assert bench.oracle_sample_shape(WORKLOADS["omni3b-b1"]) == (12, 1)
    assert bench.oracle_sample_shape(WORKLOADS["tiny"]) == (1, 1)


def test_one_core_context_restores_affinity():
    before = os.sched_getaffinity(0)
    with bench.OneCore():
        assert len(os.sched_getaffinity(0)) == 1
    assert os.sched_getaffinity(0) == before


def test_peak_source():
    peak, kind = bench.peaks()
    assert peak > 0 and kind in ("measured", "fallback")
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured"
