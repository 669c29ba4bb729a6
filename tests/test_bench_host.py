"""Host-side logic of bench.py that needs no GPU: the `config` object both
arms print, the clock-sample summary that decides whether a run was
throttled, the per-kernel DRAM traffic lookup keyed to the kernels' source
hashes, and the peak denominators."""
import argparse
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _args(workload, ep="peer", fmt="mxfp8", eager=False):
    return argparse.Namespace(workload=workload, seed=0, fmt=fmt, eager=eager, ep=ep)


@pytest.mark.parametrize("workload", ["pr1", "page", "large", "contiguous", "masked"])
def test_run_config_single_and_replicas(workload):
    one = bench.run_config(_args(workload), 1)
    assert one["parallelism"] == "single GPU"
    assert one["workload"] == workload and one["format"] == "mxfp8" and one["graph"] is True
    assert "flushed" in one["l2"]
    two = bench.run_config(_args(workload), 2)
    assert two["parallelism"] == "replicas x2"
    assert {k: v for k, v in two.items() if k != "parallelism"} == {k: v for k, v in one.items() if k != "parallelism"}


@pytest.mark.parametrize("mode,text", [("peer", "peer memory"), ("nccl", "NCCL all-to-all")])
def test_run_config_expert_parallel(mode, text):
    old = dict(bench.EP_CTX)
    try:
        bench.EP_CTX.update(world=4, rank=0, mode=mode)
        cfg = bench.run_config(_args("moe_layer_ep", ep=mode), 4)
    finally:
        bench.EP_CTX.clear()
        bench.EP_CTX.update(old)
    assert cfg["parallelism"] == f"expert parallel x4 ({text})"
    assert cfg["workload"] == "moe_layer_ep"


def test_run_config_eager_and_format():
    cfg = bench.run_config(_args("large", fmt="tilewise", eager=True), 1)
    assert cfg["graph"] is False and cfg["format"] == "tilewise"


def _line(sm, mx, power, reasons=("Not Active",) * 4):
    return f"0, {sm}, {mx}, {power}, 0x0, " + ", ".join(reasons)


def test_clock_summary_window_median_and_reasons():
    cs = bench.ClockSampler(0)
    cs.lines = [
        (0.0, _line(1965, 1965, 300.0)),                                    # before the window
        (1.0, _line(1500, 1965, 990.0, ("Not Active", "Not Active", "Not Active", "Active"))),
        (1.2, _line(1600, 1965, 995.0)),
        (1.4, _line(1700, 1965, 1000.5, ("Not Active", "Not Active", "Not Active", "Active"))),
        (1.5, "garbage line"),                                              # skipped
        (1.6, "0, N/A, 1965, 1000, 0x0, a, b, c, d"),                       # unparsable clock: skipped
        (9.0, _line(1965, 1965, 200.0, ("Active", "Not Active", "Not Active", "Not Active"))),  # after
    ]
    s = cs.summary(0.9, 1.5)
    assert s["sm_mhz"] == 1600 and s["sm_max_mhz"] == 1965
    assert s["power_w_max"] == 1000.5
    assert s["reasons"] == ["sw_power_cap"]          # hw_slowdown outside the window is not counted
    assert s["samples"] == 3 and s["samples_in_timed_region"] == 3


def test_clock_summary_falls_back_to_all_samples_and_reports_none():
    cs = bench.ClockSampler(0)
    cs.lines = [(5.0, _line(1965, 1965, 400.0, ("Not Active", "Active", "Not Active", "Not Active")))]
    s = cs.summary(0.0, 1.0)                         # no sample inside: every sample is used
    assert s["sm_mhz"] == 1965 and s["reasons"] == ["hw_thermal_slowdown"]
    assert s["samples_in_timed_region"] == 0
    empty = bench.ClockSampler(0)
    assert empty.summary(0.0, 1.0)["reasons"] == ["no nvidia-smi samples"]


def test_traffic_lookup_follows_source_hashes(monkeypatch):
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        tab = json.load(f)
    for key, ent in tab.items():
        kind, workload = key.split(":")
        want = float(ent["dram_bytes_per_launch"]) if ent["source_hash"] == bench.kernel_source_hash(kind) else None
        assert bench.lookup_traffic(kind, workload, "mxfp8") == want
    assert bench.lookup_traffic("gemm", "no_such_workload", "mxfp8") is None
    assert bench.lookup_traffic("gemm", "contiguous", "tilewise") is None   # MXFP8 captures only
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind: "0000000000000000")
    assert all(bench.lookup_traffic(*k.split(":"), "mxfp8") is None for k in tab)


def test_peaks_are_the_measured_ones():
    pk = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert pk["source"] == "measured"
        assert pk["hbm_gbs"] > 1000 and pk["bf16_tflops"] >= pk["bf16_tflops_sustained"] > 100
    else:
        assert pk["source"] == "fallback"


def test_contiguous_step_text_names_the_lean_quantisation():
    mx8 = bench.run_config(_args("contiguous"), 1)["step"]
    tw = bench.run_config(_args("contiguous", fmt="tilewise"), 1)["step"]
    assert "lean form" in mx8 and "parallel stream" in mx8
    assert "lean" not in tw
