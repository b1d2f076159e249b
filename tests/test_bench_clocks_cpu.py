"""bench.py's clock summary: only samples stamped inside the timed region count,
throttle reasons are collected from those, and a region shorter than the
sampling interval falls back to every sample (no GPU; synthetic nvidia-smi lines)."""
import datetime
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def _line(t, sm, reasons=()):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    flags = ["Active" if nm in reasons else "Not Active"
             for nm in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")]
    return ", ".join([ts, "0", f"{sm} MHz", "1965 MHz", "700.00 W", "0x4"] + flags)


def test_only_samples_inside_the_timed_region_count():
    import bench
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    c.t0, c.t1 = t0, t0 + 0.3
    c.out = "\n".join([
        _line(t0 - 0.5, 1965),                              # before: idle, max clock
        _line(t0 + 0.05, 1500, ["sw_power_cap"]),
        _line(t0 + 0.15, 1520, ["sw_power_cap"]),
        _line(t0 + 0.25, 1540),
        _line(t0 + 0.33, 1530),                             # one interval after the end: still counted
        _line(t0 + 1.0, 1965, ["hw_slowdown"]),             # long after: not counted
        "garbage line",
    ])
    s = c.summary()
    assert s["samples"] == 4 and s["window"] == "timed region"
    assert s["sm_mhz"] == 1525.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_short_region_falls_back_to_every_sample():
    import bench
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    c.t0, c.t1 = t0, t0 + 0.01
    c.out = "\n".join([_line(t0 - 0.2, 1700), _line(t0 + 0.5, 1900, ["sw_power_cap"])])
    s = c.summary()
    assert s["samples"] == 2 and s["window"] == "all samples"
    assert s["sm_mhz"] == 1800.0 and s["reasons"] == ["sw_power_cap"]


def test_no_sampler_output():
    import bench
    c = bench.ClockSampler(0)
    s = c.summary()
    assert s["sm_mhz"] is None and s["samples"] == 0 and s["reasons"] == []
