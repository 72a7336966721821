"""bench.py's host-side bookkeeping (CPU, no GPU): the clock-sample summary that decides
whether a timed run was throttled, and the roofline denominators and traffic lookup."""
import json

import pytest

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


def test_traffic_is_reported_only_for_its_workload_kernel_and_build(tmp_path, monkeypatch):
    from recurrent_vision_backbone_only_b200 import build
    p = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    entry = {"workload": "gtr640", "kernel": "tensor-core 128-row",
             "lib_sources_digest": build.sources_digest(), "dram_bytes_per_launch": 123456}
    p.write_text(json.dumps({"entries": [entry]}))
    assert bench.profile_traffic("gtr640", "tensor-core 128-row") == 123456
    assert bench.profile_traffic("highres", "tensor-core 128-row") is None
    assert bench.profile_traffic("gtr640", "tensor-core 64-row pipelined") is None
    p.write_text(json.dumps({"entries": [dict(entry, lib_sources_digest="0" * 16)]}))
    assert bench.profile_traffic("gtr640", "tensor-core 128-row") is None   # kernel changed since
    p.unlink()
    assert bench.profile_traffic("gtr640", "tensor-core 128-row") is None


NCU_DETAILS = """==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(192, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","206.02"
"0","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(192, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Mbyte","29.07"
"2","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(132, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","50"
"2","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(132, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Mbyte","10"
"3","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(192, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","206.02"
"3","1","python","h","void gla::ck::gla_pipe_kernel(Maps, Params)","1","7","(576, 1, 1)","(192, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Mbyte","29.07"
"1","1","python","h","void other_kernel()","1","7","(1, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","7"
"1","1","python","h","void other_kernel()","1","7","(1, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","0"
"""


def test_ncu_csv_reader_and_traffic_entry(tmp_path, capsys):
    p = tmp_path / "n.csv"
    p.write_text(NCU_DETAILS)
    got = bench.read_ncu_csv(str(p))
    assert [k for k, _ in got][:2] == ["void gla::ck::gla_pipe_kernel(Maps, Params)"] * 2
    assert got[0][1]["dram__bytes_read.sum"] == pytest.approx(206.02e6)
    assert got[1][1]["grid"] == "(132, 1, 1)"
    args = bench.argparse.Namespace(record_traffic=str(p), workload="batched", kernel="pipe64",
                                    ncu_command="ncu ...")
    bench.record_traffic(args)
    e = json.loads(capsys.readouterr().out)
    assert e["workload"] == "batched" and e["kernel"] == "tensor-core 64-row pipelined"
    # a call = one launch of each grid shape: (206.02 + 29.07) + (50 + 10) MB
    assert e["dram_bytes_per_launch"] == pytest.approx(295.09e6)
    assert e["launches"] == 3 and len(e["launch_shapes"]) == 2


def test_gate_bytes_and_traffic_entry(tmp_path, capsys):
    from recurrent_vision_backbone_only_b200 import synth
    wl = synth.WORKLOADS["batched"]
    assert bench.gate_shape(wl, 384) == (16 * 1600, 384, 12 * 64)
    # x read once, a written once (fp16), W1 / W2 (fp16) and b (fp32) read once
    assert bench.gate_bytes(wl, 384) == 25600 * 384 * 2 + 25600 * 768 * 2 + 16 * 384 * 2 \
        + 16 * 768 * 2 + 768 * 4
    csv = NCU_DETAILS.replace("void gla::ck::gla_pipe_kernel(Maps, Params)",
                              "void gla::gp::gla_gate_kernel(CUtensorMap_st, GateParams)")
    p = tmp_path / "g.csv"
    p.write_text(csv)
    args = bench.argparse.Namespace(record_traffic=str(p), workload="batched", kernel="auto",
                                    op="gate", d_model=384, ncu_command="ncu ...")
    bench.record_traffic(args)
    e = json.loads(capsys.readouterr().out)
    assert e["kernel"] == bench.GATE_KERNEL and e["launches"] == 3
    # one launch per call: the mean over launches
    assert e["dram_bytes_per_launch"] == pytest.approx((2 * 235.09e6 + 60e6) / 3)
    assert e["algorithmic_bytes_per_launch"] == bench.gate_bytes(wl, 384)


def test_sswiglu_bytes():
    from recurrent_vision_backbone_only_b200 import synth
    wl = synth.WORKLOADS["gtr640"]
    C = 4 * 384
    # value and gate read, h written (fp16); 9 taps and a bias (fp32) per channel
    assert bench.sswiglu_bytes(wl, 384) == 3 * 2 * 1600 * C + 4 * 10 * C


def test_linear_bytes_and_bound_inputs():
    # x read, y written, W read once (fp16)
    assert bench.linear_bytes(1600, 384, 1536) == 2 * (1600 * 384 + 1600 * 1536 + 384 * 1536)
    tpeak, kind = bench.measured_tensor_peak()
    assert tpeak > 100 and kind in ("measured", "fallback")


def test_aux_roofline_picks_the_binding_roof():
    hbm, tensor = (6545.9, "measured"), (1609.7, "measured")
    # the batched input projections: 60.4 GFLOP need 37.5 us on the tensor roof, 179 MB need
    # 27.4 us on the HBM roof -> tensor-bound
    r = bench.aux_roofline(179_306_496, 60_397_977_600, 74.8e-6, hbm, tensor)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(60_397_977_600 / 74.8e-6 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1609.7)
    assert r["hbm_frac"] == pytest.approx(179_306_496 / 74.8e-6 / 1e9 / 6545.9)
    # the 40x40 B=1 output projection: 0.47 GFLOP vs 2.5 MB -> HBM-bound
    r = bench.aux_roofline(2_752_512, 471_859_200, 7.28e-6, hbm, tensor)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["flops_per_launch"] == 471_859_200
    # no FLOPs given (gate, Spatial SwiGLU): HBM, no tensor keys
    r = bench.aux_roofline(59_022_336, 0, 17.42e-6, hbm, tensor)
    assert r["bound"] == "hbm" and "flops_per_launch" not in r
    assert r["frac"] == pytest.approx(59_022_336 / 17.42e-6 / 1e9 / 6545.9)
