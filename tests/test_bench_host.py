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


@pytest.mark.parametrize("workload", ["contiguous", "large"])
def test_step_text_names_the_lean_quantisation(workload):
    mx8 = bench.run_config(_args(workload), 1)["step"]
    tw = bench.run_config(_args(workload, fmt="tilewise"), 1)["step"]
    assert "lean form" in mx8 and "parallel stream" in mx8
    assert "lean" not in tw


class _FakeCuda:
    """Stand-ins for the torch.cuda stream/event calls run_eager makes,
    recording the order in which launches, waits and records are issued on
    which stream."""

    def __init__(self):
        self.log = []
        self.current = None
        self.main = self.Stream(self, "main")

    class Stream:
        def __init__(self, fc, name=None, device=None):
            self.fc, self.name = fc, name or f"side{len([e for e in fc.log if e[0] == 'new'])}"
            fc.log.append(("new", self.name))

        def wait_stream(self, other):
            self.fc.log.append(("wait_stream", self.name, other.name))

        def wait_event(self, ev):
            assert ev.recorded, "waiting on an event that was never recorded"
            self.fc.log.append(("wait_event", self.name, ev.tag))

    class Event:
        def __init__(self, fc):
            self.fc, self.recorded, self.tag = fc, False, None

        def record(self, stream):
            self.recorded, self.tag = True, stream.fc.current_launch
            self.fc.log.append(("record", stream.name, self.tag))


def test_run_eager_branch_waits(monkeypatch):
    import contextlib
    import torch
    fc = _FakeCuda()
    fc.current = fc.main
    fc.current_launch = None

    @contextlib.contextmanager
    def stream_ctx(st):
        prev, fc.current = fc.current, st
        try:
            yield
        finally:
            fc.current = prev

    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: fc.current)
    monkeypatch.setattr(torch.cuda, "Stream", lambda device=None: _FakeCuda.Stream(fc, device=device))
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeCuda.Event(fc))
    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)

    def launch(i):
        def fn():
            fc.current_launch = i
            fc.log.append(("launch", fc.current.name, i))
        return ("quant", f"l{i}", fn, 0.0, 0.0, ())

    wl = object.__new__(bench.Workload)
    wl.dev = "cpu"
    wl._side = []
    # the large workload's shape: 0 quantise, 1 and 2 lean quantisations, 3..5 GEMMs
    wl.launches = [launch(i) for i in range(6)]
    wl.branches = [[0, 3, 4, 5], [1, 2]]
    wl.waits = {4: [1], 5: [2]}
    wl.after = []
    wl.run_eager()
    log = fc.log
    launches = [e for e in log if e[0] == "launch"]
    assert sorted(e[2] for e in launches) == list(range(6))
    on = {e[2]: e[1] for e in launches}
    assert on[0] == on[3] == on[4] == on[5] == "main" and on[1] == on[2] != "main"
    pos = {e[2]: k for k, e in enumerate(log) if e[0] == "launch"}
    for i, deps in wl.waits.items():
        for d in deps:
            rec = next(k for k, e in enumerate(log) if e[0] == "record" and e[2] == d)
            wait = next(k for k, e in enumerate(log) if e[0] == "wait_event" and e[2] == d and e[1] == on[i])
            assert pos[d] < rec < wait < pos[i]
    assert pos[3] < pos[4] < pos[5] and pos[0] < pos[3] and pos[1] < pos[2]
    # the side stream forks from and joins back into the main stream
    side = on[1]
    fork = next(k for k, e in enumerate(log) if e == ("wait_stream", side, "main"))
    join = next(k for k, e in enumerate(log) if e == ("wait_stream", "main", side))
    assert fork < pos[1] and join > max(pos.values())

    # the contiguous workload's shape: a launch after the join
    fc.log.clear()
    wl.launches = [launch(i) for i in range(4)]
    wl.branches = [[0, 2], [1]]
    wl.waits = {}
    wl.after = [3]
    wl.run_eager()
    log = fc.log
    pos = {e[2]: k for k, e in enumerate(log) if e[0] == "launch"}
    join = next(k for k, e in enumerate(log) if e[0] == "wait_stream" and e[1] == "main")
    assert join < pos[3] and all(pos[i] < join for i in range(3))
