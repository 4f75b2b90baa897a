"""bench.py's clock record: samples are kept only inside the timed region when it is
marked, throttle reasons are collected from the samples kept, and the whole sampling
period (its loaded part) is the fallback when no sample falls inside."""
import datetime
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _line(t, sm, power_cap=False, thermal=False):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    act = lambda b: "Active" if b else "Not Active"  # noqa: E731
    return (f"{ts}, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, {act(thermal)}, "
            f"{act(power_cap)}\n")


T0 = 1_800_000_000.0
LINES = ([_line(T0 + 0.05 * i, 1965) for i in range(6)]                      # idle, before
         + [_line(T0 + 0.3 + 0.05 * i, 1650 + i, power_cap=True) for i in range(5)]
         + [_line(T0 + 0.6, 1965, thermal=True), "garbage line\n"])           # after


def test_window_keeps_only_the_timed_region():
    kept = bench.ClockSampler.parse(LINES, (T0 + 0.29, T0 + 0.51))
    assert [x[1] for x in kept] == [1650, 1651, 1652, 1653, 1654]
    out = bench.ClockSampler.summarise(kept, True)
    assert out["sm_mhz"] == 1652 and out["sm_min_mhz"] == 1650 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 5
    assert out["window"] == "timed region"


def test_fallback_to_the_loaded_samples():
    allp = bench.ClockSampler.parse(LINES)
    assert len(allp) == 12
    out = bench.ClockSampler.summarise(allp, False)
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert out["window"] == "whole sampling period"
    assert bench.ClockSampler.summarise([], True)["samples"] == 0


def test_untimestamped_samples_are_never_inside_a_window():
    bad = ["n/a, 1700, 1965, 700, 0x0, Not Active, Not Active, Not Active, Active\n"]
    assert bench.ClockSampler.parse(bad, (0, 1e12)) == []
    assert len(bench.ClockSampler.parse(bad)) == 1
