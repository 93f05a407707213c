"""bench.py's clock record (host logic, no GPU): samples inside the timed region only, the median SM clock,
the throttle reasons seen active, and a record that says so when nothing was sampled."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler(rows):
    s = bench.ClockSampler.__new__(bench.ClockSampler)  # no nvidia-smi process: samples are injected
    s.samples = rows
    s.proc = None
    return s


def _row(sm, power="400.0", hw="Not Active", hw_th="Not Active", sw_th="Not Active", cap="Not Active"):
    # fields in ClockSampler.FIELDS order: timestamp, index, clocks.sm, clocks.max.sm, power.draw, active mask,
    # hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    return ["2026/12/02 10:00:00.000", "0", sm, "1965", power, "0x0", hw, hw_th, sw_th, cap]


def test_summary_takes_the_median_inside_the_region_and_the_active_reasons():
    rows = [(0.5, _row("900")),                       # before the timed region: ignored
            (1.0, _row("1965")), (1.1, _row("1950", power="612.5")), (1.2, _row("1965", cap="Active")),
            (2.5, _row("800", hw="Active"))]          # after it: ignored
    s = _sampler(rows).summary(1.0, 1.2)
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] == 612.5


def test_summary_reports_the_throttles_that_reject_a_run():
    rows = [(1.0, _row("1500", hw_th="Active")), (1.05, _row("1400", sw_th="Active", hw="Active"))]
    s = _sampler(rows).summary(1.0, 1.05)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1450.0


def test_summary_skips_unreadable_fields():
    rows = [(1.0, _row("[N/A]", power="[N/A]")), (1.01, _row("1965"))]
    s = _sampler(rows).summary(1.0, 1.01)
    assert s["sm_mhz"] == 1965.0 and s["samples"] == 2


def test_no_sample_inside_the_region_is_stated():
    s = _sampler([(0.1, _row("1965"))]).summary(1.0, 2.0)
    assert s["samples"] == 0 and s["sm_mhz"] is None
    assert s["reasons"] == ["no sample inside the timed region"]
