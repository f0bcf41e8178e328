"""Host logic of the benchmark's clock record, on CPU: only nvidia-smi samples
taken inside the timed region count, the throttle reasons seen there are
reported, and malformed lines are skipped."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _line(t, mhz, power, cap="Not Active", hw="Not Active"):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{ts}, 0, {mhz}, 1965, {power}, 0x0, {hw}, Not Active, Not Active, {cap}"


def test_only_samples_inside_the_timed_region_count():
    t0 = 1_800_000_000.0
    lines = [_line(t0 - 0.2, 1965, 120.0),              # idle, before the region
             _line(t0 + 0.02, 1500, 950.0, cap="Active"),
             _line(t0 + 0.04, 1520, 960.0, cap="Active"),
             _line(t0 + 0.06, 1600, 940.0),
             _line(t0 + 0.5, 1965, 110.0, hw="Active"),  # after the region
             "not a sample", ""]
    r = bench.ClockSampler.parse(lines, t0, t0 + 0.1)
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1520.0
    assert r["power_w"] == 950.0
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]          # the hw_slowdown sample lies outside


def test_no_sample_in_the_region():
    r = bench.ClockSampler.parse([_line(1_800_000_000.0, 1965, 100.0)], 1_900_000_000.0, 1_900_000_001.0)
    assert r["samples"] == 0 and r["sm_mhz"] is None and r["reasons"] == []
