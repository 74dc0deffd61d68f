"""bench.py's host-side measurement rules, on the CPU: the DRAM traffic of a
committed ncu summary is reported only while the kernel sources hash to the
captured ones, and the clock record keeps the samples taken inside the timed
window, their median SM clock and every throttle reason seen there."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _summary_with(tmp_path, sha, dram):
    p = tmp_path / "summary.txt"
    p.write_text(f"command: ncu ...\nsources_sha256: {sha}\ndram_bytes_per_launch: {dram}\n")
    return str(p)


def test_gemm_traffic_is_dropped_when_the_sources_changed(tmp_path, monkeypatch):
    good = _summary_with(tmp_path, bench.gemm_sources_sha256(), 12345)
    monkeypatch.setattr(bench, "GEMM_PROFILE", good)
    assert bench.gemm_dram_traffic() == 12345
    stale = _summary_with(tmp_path, "0" * 64, 12345)
    monkeypatch.setattr(bench, "GEMM_PROFILE", stale)
    assert bench.gemm_dram_traffic() is None
    monkeypatch.setattr(bench, "GEMM_PROFILE", str(tmp_path / "missing.txt"))
    assert bench.gemm_dram_traffic() is None


def test_quantize_traffic_is_dropped_when_the_sources_changed(tmp_path, monkeypatch):
    stale = _summary_with(tmp_path, "f" * 64, 999)
    monkeypatch.setattr(bench, "QUANT_PROFILE", stale)
    assert bench.quantize_dram_traffic() is None


def _line(sm, sm_max, hw=False, thermal=False, power=False):
    act = lambda b: "Active" if b else "Not Active"  # noqa: E731
    return f"{sm}, {sm_max}, 700.0, 0x0, {act(hw)}, {act(thermal)}, Not Active, {act(power)}"


def test_clock_summary_keeps_the_window_and_its_reasons():
    s = bench.ClockSampler(0)
    s.lines = [(1.0, _line(1000, 1965, hw=True)),       # before the window
               (2.0, _line(1965, 1965)),
               (2.1, _line(1950, 1965, power=True)),
               (2.2, _line(1965, 1965)),
               (3.0, _line(800, 1965, thermal=True)),   # after it
               (2.15, "garbage line")]
    c = s.summary(1.5, 2.5)
    assert c["samples"] == 3 and c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    whole = s.summary()
    assert whole["samples"] == 5
    assert set(whole["reasons"]) == {"hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"}


def test_clock_summary_without_samples_says_so():
    s = bench.ClockSampler(0)
    c = s.summary(0.0, 1.0)
    assert c["samples"] == 0 and c["sm_mhz"] is None and c["reasons"] == ["no nvidia-smi samples"]
