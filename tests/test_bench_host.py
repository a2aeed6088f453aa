"""bench.py's host-side bookkeeping, on CPU: the clock-sample summary, the committed DRAM-traffic
records and the fallback peak."""
import glob
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synth import workloads  # noqa: E402


def _summary(lines):
    s = bench.ClockSampler(0)
    s.file.write("".join(line + "\n" for line in lines))
    return s.summary()


def test_clock_summary_median_max_and_reasons():
    na, act = "Not Active", "Active"
    rows = [f"0, {mhz}, 1965, 800.0, 0x0, {na}, {na}, {na}, {cap}"
            for mhz, cap in ((1965, na), (1800, act), (1900, na), (1300, act), (1950, na))]
    out = _summary(rows + ["garbage line", "0, [N/A], 1965, 1, 0, a, b, c, d"])
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965 and out["samples"] == 5
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_thermal_slowdown():
    out = _summary(["0, 1500, 1965, 900.0, 0x60, Not Active, Active, Active, Not Active"])
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_says_unavailable():
    assert _summary([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}


TRAFFIC = os.path.join(ROOT, "profiles", "engine_kernel_traffic.json")


def test_traffic_record_is_consistent():
    """The committed DRAM record of the one-layer profiling case: read + write = per-step traffic;
    its algorithmic bytes are the workload's active bytes at the captured step (context + 3
    warm-up steps + half of 2 timed steps, as its command runs it); traffic exceeds them by
    less than 2 %."""
    with open(TRAFFIC) as f:
        d = json.load(f)
    assert d["dram_bytes_read"] + d["dram_bytes_write"] == d["dram_bytes_per_step"]
    w = workloads.get(d["workload"])
    assert "--steps 2 --warmup 3" in d["command"] and "--clock-control none" in d["command"]
    assert f"--workload {d['workload']}" in d["command"]
    assert workloads.active_bytes_per_token(w, w["ctx"] + 4)["total"] == d["algorithmic_bytes_per_step"]
    assert 1.0 <= d["dram_bytes_per_step"] / d["algorithmic_bytes_per_step"] < 1.02


def test_recorded_traffic_needs_the_matching_source(monkeypatch):
    with open(TRAFFIC) as f:
        d = json.load(f)
    ratio = d["dram_bytes_per_step"] / d["algorithmic_bytes_per_step"]
    monkeypatch.setattr(bench, "source_hash", lambda: d["source_hash"])
    assert bench.recorded_traffic(8e9) == pytest.approx(8e9 * ratio)
    for x in d.get("same_kernel_sources", []):
        monkeypatch.setattr(bench, "source_hash", lambda: x["source_hash"])
        assert bench.recorded_traffic(8e9) == pytest.approx(8e9 * ratio)
    monkeypatch.setattr(bench, "source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic(8e9) is None


def test_peak_fallback_without_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6450.5}))
    assert bench.measured_peaks() == (6450.5, "measured")


def test_l2_note_tells_streaming_from_warm_steps():
    from synth import workloads as wl
    big = wl.active_bytes_per_token(wl.get("moe_mla_fp8_1k"), 1024)["total"]
    tiny = wl.active_bytes_per_token(wl.get("tiny_dense_f32"), 64)["total"]
    assert "far above" in bench.l2_note(big)
    assert "warm" in bench.l2_note(tiny) and "far above" not in bench.l2_note(tiny)
