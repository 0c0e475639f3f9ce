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


def test_measured_peaks_are_read_whatever_the_file_holds(tmp_path, monkeypatch):
    """The roofline denominators come from MEASURED_PEAKS.json when it holds usable
    numbers (plain or as an object's "value"), and fall back to the pool's earlier
    measurement for a missing file, a missing key or a value that is not a number."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._peaks() == (bench.FALLBACK_HBM_GBS, 1965.0, "fallback")
    assert bench._tensor_peak_tflops() == 1590.0
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text(json.dumps({"hbm_gbs": 6547.2, "bf16_tflops": 1585.0}))
    assert bench._peaks() == (6547.2, 1965.0, "measured")
    assert bench._tensor_peak_tflops() == 1585.0
    f.write_text(json.dumps({"hbm_gbs": {"value": 6500.0}, "bf16_tflops": {"burst": 1}, "sm_max_mhz": 1965}))
    assert bench._peaks() == (6500.0, 1965.0, "measured")
    assert bench._tensor_peak_tflops() == 1590.0
    f.write_text(json.dumps({"hbm_gbs": [1, 2]}))
    assert bench._peaks()[2] == "fallback"
    f.write_text("not json")
    assert bench._peaks()[2] == "fallback"
