"""CPU checks of the benchmark's host-side pieces: the clock-sample summary that
goes into the JSON line, the algorithmic byte count behind the roofline, the
whole-job throughput, and the CPU description."""
import datetime

import bench
import pn_inputs as pi


def _line(ts, mhz, reasons=("Not Active",) * 4, max_mhz=1965):
    stamp = datetime.datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([stamp, str(mhz), str(max_mhz), *reasons])


def test_clock_summary_uses_samples_inside_the_timed_region():
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    c.t0, c.t1 = t0 + 1.0, t0 + 2.0
    c.lines = [_line(t0 + 0.5, 900, ("Active", "Not Active", "Not Active", "Not Active")),   # before: ignored
               _line(t0 + 1.2, 1900),
               _line(t0 + 1.4, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
               _line(t0 + 1.6, 1800),
               _line(t0 + 2.5, 500, ("Not Active", "Active", "Not Active", "Not Active")),      # after: ignored
               "garbage line"]
    s = c.summary()
    assert s["samples"] == 3 and not s["nearest_used"]
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_the_nearest_samples():
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    c.t0, c.t1 = t0 + 1.000, t0 + 1.005          # shorter than the sampling period
    c.lines = [_line(t0 + 0.99, 1950), _line(t0 + 1.02, 1960), _line(t0 + 3.0, 100)]
    s = c.summary()
    assert s["samples"] == 0 and s["nearest_used"] and s["sm_mhz"] == 1955


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 1.0, 2.0
    s = c.summary()
    assert s["sm_mhz"] is None and s["reasons"] == [] and s["samples"] == 0


def test_algorithmic_bytes_of_the_headline_workload():
    p = pi.benchmark_workload(1, T=64, B=2)      # same D and cell as the full size
    # read u_t and s^(i)_t, write s^(i+1)_t: 3 * 64 floats per (b, t)
    assert bench.alg_bytes_per_step(p) == 4 * (64 + 2 * 64)
    assert bench.alg_bytes_per_step(p) * 16 * 16384 == 201_326_592
    g = pi.benchmark_workload(3, T=64, B=2)      # GRU: three gate inputs per step
    assert bench.alg_bytes_per_step(g) == 4 * (3 * 32 + 2 * 32)


def test_job_throughput_and_cpu_model():
    assert bench.job_throughput(1000.0, 4, 2.0) == 2_000_000.0
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def test_traffic_only_while_the_device_source_matches(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu figure only while the device code hashes to the
    value recorded beside it; any other source, an unknown workload or no file gives None."""
    import json
    p = pi.benchmark_workload(1, T=64, B=2)
    key = f"{p.name}:{pi.MODE_NAMES[pi.MODE_QUASI]}"
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.traffic_from_profile(p, pi.MODE_QUASI) is None          # no file
    sha = bench.kernel_source_sha()
    (tmp_path / "traffic.json").write_text(json.dumps({key: {"source_sha": sha, "dram_bytes_per_launch": 1.5e8}}))
    assert bench.traffic_from_profile(p, pi.MODE_QUASI) == 1.5e8
    assert bench.traffic_from_profile(p, pi.MODE_JACOBI) is None         # no entry for that mode
    (tmp_path / "traffic.json").write_text(json.dumps({key: {"source_sha": "0" * 16, "dram_bytes_per_launch": 1.5e8}}))
    assert bench.traffic_from_profile(p, pi.MODE_QUASI) is None          # taken on another source
