"""Host logic of bench.py: the nvidia-smi clock-sample parser, the sampler
where nvidia-smi cannot run, and the traffic record keyed to a source file
(no GPU needed)."""
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


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    """roofline.traffic comes from an ncu capture of a kernel's source file;
    once the file differs from the captured one it must read as unknown."""
    import hashlib
    src = tmp_path / "kernel.cu"
    src.write_text("// captured version\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURES", {("w", "k"): {"bytes": 123, "source": "kernel.cu",
                                                                 "sha256": digest, "profile": "p.md"}})
    assert bench.captured_traffic("w", "k") == 123
    assert bench.captured_traffic("w", "other") is None
    src.write_text("// changed since the capture\n")
    assert bench.captured_traffic("w", "k") is None
    src.unlink()
    assert bench.captured_traffic("w", "k") is None
