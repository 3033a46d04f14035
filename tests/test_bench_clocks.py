"""The bench's summary of the nvidia-smi samples taken during a timed region
(no GPU: fixed sample lines): median SM clock, max clock, active throttle
reasons, and only the lines of the benchmarked GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

A, B = "GPU-aaaa", "GPU-bbbb"


def line(uuid, sm, smax=1965, active="0x0", hw="Not Active", hwt="Not Active", swt="Not Active", pcap="Not Active"):
    return f"{uuid}, {sm}, {smax}, 612.3, {active}, {hw}, {hwt}, {swt}, {pcap}"


def test_median_and_reasons_of_this_gpu_only():
    lines = [line(A, 1965), line(A, 1950, pcap="Active"), line(A, 1965), line(B, 300, hw="Active"),
             "garbage", line(A, "[N/A]")]
    d = bench.ClockSampler.summarize(lines, A)
    assert d == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_slowdown_reasons_are_reported():
    lines = [line(A, 1200, hw="Active"), line(A, 1100, hwt="Active", swt="Active")]
    d = bench.ClockSampler.summarize(lines, A)
    assert d["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert d["sm_mhz"] == 1150.0


def test_no_samples_gives_none():
    assert bench.ClockSampler.summarize([], A) is None
    assert bench.ClockSampler.summarize([line(B, 1965)], A) is None
    assert bench.ClockSampler.summarize([line(B, 1965)], "")["samples"] == 1
