"""The clock record of the bench line, parsed from nvidia-smi's CSV (no GPU needed): the median
SM clock under load, the maximum, and which throttle reasons were active at any sample."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler_with(lines, tmp_path):
    s = bench.ClockSampler(0)
    p = tmp_path / "clocks.csv"
    p.write_text("".join(l + "\n" for l in lines))
    s.path = str(p)
    return s


def test_power_cap_is_reported_and_median_taken(tmp_path):
    lines = [
        "0, 1965, 1965, 640.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1755, 1965, 1001.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    ]
    c = _sampler_with(lines, tmp_path).summary()
    assert c["sm_mhz"] == 1800 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3


def test_thermal_and_hardware_slowdown_are_named(tmp_path):
    lines = [
        "0, 1500, 1965, 700.0, 0x0000000000000048, Active, Not Active, Active, Not Active",
        "0, 1400, 1965, 700.0, 0x0000000000000040, Not Active, Active, Not Active, Not Active",
    ]
    c = _sampler_with(lines, tmp_path).summary()
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_samples_reads_unavailable(tmp_path):
    c = _sampler_with(["garbage"], tmp_path).summary()
    assert c["sm_mhz"] is None and c["reasons"] == ["unavailable"]
