"""bench.py's clock record: the median SM clock under load, the maximum clock
and every clock-event reason seen in any sample (hw_slowdown and the thermal
reasons reject a run; sw_power_cap is kept and noted).  Host only."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler(lines):
    c = bench.ClockSampler(0)
    c.lines = list(lines)
    return c.summary()


def test_median_max_and_reasons():
    s = _sampler(["1900, 1965, 800.0, 0x4, Not Active, Not Active, Not Active, Active",
                  "1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                  "1850, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active"])
    assert s == {"sm_mhz": 1850.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_rejecting_reasons_are_reported():
    s = _sampler(["1200, 1965, 700.0, 0x48, Active, Active, Not Active, Not Active",
                  "1250, 1965, 700.0, 0x20, Not Active, Not Active, Active, Not Active"])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_samples_and_malformed_lines():
    assert _sampler([])["samples"] == 0
    assert _sampler(["[N/A], [N/A], [N/A], 0x0, Not Active, Not Active, Not Active, Not Active", "garbage"]) == \
        {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_reason_bits_follow_the_field_order():
    # NVML bits for hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    assert bench.ClockSampler.REASON_BITS == (0x8, 0x40, 0x20, 0x4)
    assert bench.ClockSampler.FIELDS.split(",")[4:] == [
        "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
        "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
