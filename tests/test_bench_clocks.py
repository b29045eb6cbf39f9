"""Host logic of bench.py's clock record: the nvidia-smi sample parser and
the sampler's behaviour where nvidia-smi cannot run (no GPU needed)."""
import os
import tempfile

import bench


def test_clock_summary_parses_samples_and_reasons():
    c = bench.ClockSampler(0, None)
    c.text = "\n".join([
        "0, 1965, 1965, 700.1, 0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle: ignored
        "0, 1900, 1965, 900.5, 100, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 990.0, 100, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 995.0, 97, 0x4, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_thermal_slowdown():
    c = bench.ClockSampler(0, None)
    c.text = "0, 1500, 1965, 900, 100, 0x20, Not Active, Not Active, Active, Not Active"
    assert bench.ClockSampler.summary(c)["reasons"] == ["sw_thermal_slowdown"]


def test_clock_sampler_without_samples():
    path = os.path.join(tempfile.gettempdir(), f"la_bench_clock_test_{os.getpid()}.csv")
    with bench.ClockSampler(0, path) as c:
        pass   # no timed work; here nvidia-smi may be missing altogether
    s = c.summary()
    assert s["samples"] >= 0 and isinstance(s["reasons"], list)
    if os.path.exists(path):
        os.remove(path)
