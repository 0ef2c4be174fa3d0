"""The clock record of bench.py's timed region: NVML samples (SM clock,
throttle-reason bit mask) reduced to the median clock under load, the
maximum clock and the reasons that were active inside the region."""
import bench


def _sampler(max_mhz=1965.0):
    s = object.__new__(bench.NvmlSampler)  # no NVML on the CPU: only the summary
    s.max_mhz = max_mhz
    return s


def test_summary_keeps_only_the_timed_region():
    s = _sampler()
    rows = [(0.5, 120.0, 0x1), (1.0, 1965.0, 0x0), (1.01, 1950.0, 0x4), (1.02, 1965.0, 0x0),
            (2.5, 900.0, 0x40)]
    got = s.summarize(rows, 1.0, 2.0)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1965.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]   # the thermal sample lies outside


def test_summary_names_every_rejecting_reason():
    s = _sampler()
    rows = [(1.0, 1500.0, 0x8 | 0x20), (1.1, 1400.0, 0x40)]
    got = s.summarize(rows, 0.0, 2.0)
    assert got["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_summary_without_samples():
    got = _sampler().summarize([], 0.0, 1.0)
    assert got["samples"] == 0 and got["sm_mhz"] is None
