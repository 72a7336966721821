"""bench.py's host-side bookkeeping (CPU, no GPU): the clock-sample summary that decides
whether a timed run was throttled, and the roofline denominators and traffic lookup."""
import json

import bench


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.out = "\n".join(lines)
    return s


def test_clock_summary_median_max_and_no_reason():
    rows = ["0, 1965, 1965, 410.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
            "0, 1950, 1965, 420.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
            "0, 1965, 1965, 430.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"]
    s = _sampler(rows).summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == [] and s["samples"] == 3


def test_clock_summary_names_each_active_reason_once():
    rows = ["0, 1300, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "0, 1290, 1965, 995.0, 0x0000000000000044, Not Active, Active, Not Active, Active",
            "0, 1310, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active"]
    s = _sampler(rows).summary()
    assert s["sm_mhz"] == 1300.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_summary_skips_malformed_rows_and_reports_no_samples():
    assert _sampler(["", "garbage", "0, [N/A], 1965, 1, 0x0, a, b, c, d"]).summary() == {
        "sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
    s = _sampler(["0, 1965, 1965, 400, 0x0, Not Active, Not Active, Not Active, Not Active",
                  "short, row"]).summary()
    assert s["samples"] == 1


def test_peaks_read_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6545.9}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6545.9, "measured")
    (tmp_path / "MEASURED_PEAKS.json").unlink()
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")


def test_traffic_is_reported_only_for_its_workload_and_build(tmp_path, monkeypatch):
    from recurrent_vision_backbone_only_b200 import build
    p = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    p.write_text(json.dumps({"workload": "gtr640", "lib_sources_digest": build.sources_digest(),
                             "dram_bytes_per_launch": 123456}))
    assert bench.profile_traffic("gtr640") == 123456
    assert bench.profile_traffic("highres") is None
    p.write_text(json.dumps({"workload": "gtr640", "lib_sources_digest": "0" * 16,
                             "dram_bytes_per_launch": 123456}))
    assert bench.profile_traffic("gtr640") is None          # kernel changed since the capture
    p.unlink()
    assert bench.profile_traffic("gtr640") is None
