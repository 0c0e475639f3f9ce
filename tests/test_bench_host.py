"""Host-side logic of bench.py that needs no GPU: the clock record keeps only the
samples taken inside the timed region, and reports every clock-event reason seen."""
import bench


def _sampler(samples, max_mhz=1965.0):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = samples
    s.max_mhz = max_mhz
    s.source = "test"
    return s


def test_summary_keeps_only_samples_inside_the_region():
    smp = _sampler([(0.0, 600.0, 0x1), (1.0, 1800.0, 0), (1.1, 1965.0, 0x4), (1.2, 1965.0, 0), (5.0, 600.0, 0x1)])
    rec = smp.summary(0.9, 1.25)
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1965.0 and rec["sm_min_mhz"] == 1800.0
    assert rec["reasons"] == ["sw_power_cap"]          # idle (0x1) outside the window is dropped
    assert rec["window"] == "timed region only"


def test_summary_of_a_region_shorter_than_the_period_takes_the_nearest_sample():
    smp = _sampler([(0.0, 700.0, 0), (1.0, 1900.0, 0x40)])
    rec = smp.summary(0.97, 0.98)
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1900.0
    assert rec["reasons"] == ["hw_thermal_slowdown"]


def test_summary_without_samples_is_none():
    assert _sampler([]).summary(0.0, 1.0) is None
