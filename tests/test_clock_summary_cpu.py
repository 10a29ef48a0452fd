"""bench.py's clock record, from synthetic nvidia-smi lines and NVML rows (no GPU): samples inside
the timed region are the ones reported, and every throttle reason seen there is listed."""
import importlib.util
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_for_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(b)
    finally:
        sys.argv = argv
    return b


def _fake_nvml():
    # the bit values of the real enumeration do not matter here, only that each reason has its own
    return types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
                                 nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4,
                                 nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80)


def test_summary_prefers_samples_inside_the_timed_region():
    b = _bench()
    c = b.ClockSampler(0)
    c.t_start, c.t_stop = 100.0, 101.0
    line = "0, {sm}, 1965, 300.0, 0x0, {hw}, Not Active, Not Active, {pc}"
    c.lines = [(90.0, line.format(sm=1000, hw="Active", pc="Not Active")),      # long before: ignored
               (100.5, line.format(sm=1965, hw="Not Active", pc="Active")),
               (100.9, line.format(sm=1950, hw="Not Active", pc="Not Active"))]
    out = c.summary()
    assert out["sm_mhz"] == (1965 + 1950) / 2 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample lies outside the region
    assert out["samples_in_timed_region"] == 2 and out["nvml_samples_in_timed_region"] == 0


def test_summary_takes_nvml_rows_and_their_reasons():
    b = _bench()
    c = b.ClockSampler(0)
    c.t_start, c.t_stop = 100.0, 100.01  # a region shorter than the nvidia-smi period
    c.nvml = _fake_nvml()
    c.nvml_rows = [(1965, 0x0), (1965, 0x4), (1800, 0x8)]
    out = c.summary()
    assert out["nvml_samples_in_timed_region"] == 3 and out["samples_in_timed_region"] == 3
    assert out["sm_mhz"] == 1965 and out["sm_mhz_min_in_timed_region"] == 1800
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_summary_without_any_sample():
    b = _bench()
    c = b.ClockSampler(0)
    out = c.summary()
    assert out["sm_mhz"] is None and out["samples"] == 0
