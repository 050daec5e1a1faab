"""Host logic of the benchmark that needs no GPU: argument checks, the clock
sampler's accept / reject rule (against a fake NVML), the measured-peak and
ncu-traffic records."""
import hashlib
import json
import os
import shutil
import sys
import time
import types

import numpy as np
import pytest

import bench


def test_parse_args_defaults_and_checks():
    a = bench.parse_args([])
    assert a.workload == "qwen7b_1m" and a.impl == "ours" and a.warmup >= 3 and a.layers is None
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    assert bench.parse_args(["--workload", "qwen7b_1m", "--layers", "1"]).layers == 1
    with pytest.raises(SystemExit):
        bench.parse_args(["--workload", "qwen7b_1m", "--layers", "29"])
    with pytest.raises(SystemExit):
        bench.parse_args(["--layers", "0"])


class _FakeEvent:
    def __init__(self, **kw):
        pass

    def record(self):
        pass

    def elapsed_time(self, other):
        return 1.0


@pytest.mark.parametrize("n_graphs,K,W_,inner,n_singles", [
    (1, 20, 5, 1, 16), (16, 20, 5, 1, 16), (1, 50, 5, 16, 16), (2, 37, 50, 8, 16), (4, 3, 3, 4, 16)])
def test_replay_order_matches_time_graphs(monkeypatch, n_graphs, K, W_, inner, n_singles):
    """The record pass replays exactly the steps the timed region ran."""
    ran = []

    class G:
        def __init__(self, steps):
            self.steps = steps

        def replay(self):
            ran.extend(self.steps)
    graphs = [G([j * inner + r for r in range(inner)]) for j in range(n_graphs)]
    singles = [G([j]) for j in range(n_singles)]
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda: None)
    monkeypatch.setattr(bench.torch.cuda, "Event", _FakeEvent)
    _, steps_run = bench.time_graphs(graphs, K, W_, inner, singles)
    warm, timed = bench.replay_order(n_graphs, K, W_, inner, n_singles)
    assert steps_run == K == len(timed)
    assert ran == warm + timed


def test_aggregate_is_units_over_max_time():
    assert bench.aggregate(100, 4, 2.0) == 200.0


def _fake_nvml(mask, mhz, max_mhz):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByPciBusId = lambda bus: "gpu0"
    nv.nvmlDeviceGetMaxClockInfo = lambda h, which: max_mhz
    nv.nvmlDeviceGetClockInfo = lambda h, which: mhz
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: mask
    return nv


@pytest.mark.parametrize("mask,mhz,rejected,reasons", [
    (0x0, 1965, False, []),                                   # clean run
    (0x4, 1300, False, ["sw_power_cap"]),                     # power cap: kept and noted
    (0x8, 1965, True, ["hw_slowdown"]),
    (0x40, 1965, True, ["hw_thermal_slowdown"]),
    (0x20, 1965, True, ["sw_thermal_slowdown"]),
    (0x0, 900, True, []),                                     # far below max with no reason: a clock lock
])
def test_clock_sampler_rule(monkeypatch, mask, mhz, rejected, reasons):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(mask, mhz, 1965))
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=1, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda i: props)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.02)
    s = clk.summary()
    assert s["samples"] > 0 and s["sm_mhz"] == mhz and s["sm_max_mhz"] == 1965
    assert s["reasons"] == reasons and clk.rejected() == rejected


def test_clock_sampler_without_nvml(monkeypatch):
    nv = types.ModuleType("pynvml")

    def boom():
        raise RuntimeError("no driver")
    nv.nvmlInit = boom
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.summary()["reasons"] == ["nvml unavailable"] and not clk.rejected()


def test_measured_peak_record():
    value, kind = bench.measured_hbm_peak()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            assert kind == "measured" and value == float(json.load(f)["hbm_gbs"])
    else:
        assert (value, kind) == (bench.FALLBACK_HBM_GBS, "fallback")


def test_traffic_record_follows_the_kernel_source(tmp_path):
    src = tmp_path / "kernel.cu"
    src.write_text("// a kernel\n")
    rec = {"source_sha256": hashlib.sha256(src.read_bytes()).hexdigest(),
           "per_launch_bytes": {"qwen7b_1m": 1234}}
    path = tmp_path / "record.json"
    path.write_text(json.dumps(rec))
    # the record counts only while the kernel source is the one it was taken on
    assert bench.profile_traffic(str(src), "qwen7b_1m", str(path)) == 1234
    assert bench.profile_traffic(str(src), "no_such_workload", str(path)) is None
    assert bench.profile_traffic(str(src), "qwen7b_1m", str(tmp_path / "missing.json")) is None
    with open(src, "a") as f:
        f.write("// changed\n")
    assert bench.profile_traffic(str(src), "qwen7b_1m", str(path)) is None
    # the committed record, where there is one, names the dominant kernel's source
    if os.path.exists(bench.TRAFFIC_RECORD):
        with open(bench.TRAFFIC_RECORD) as f:
            assert json.load(f)["source"].endswith("score.cu")


def test_all_core_oracle_baseline_runs_threads_in_parallel():
    """The all-core CPU baseline runs the unchanged oracle on several threads;
    with two threads it completes more layer-steps per second than with one
    (the C calls release the interpreter lock)."""
    import types as _t

    import workloads as W
    cfg = W.CONFIGS["tiny"]
    wl = _t.SimpleNamespace(cfg=cfg, layers=[W.layer_inputs(cfg, 0, "cpu")])
    one = bench.cpu_baseline_all_cores(wl, 1.0, threads=1)
    two = bench.cpu_baseline_all_cores(wl, 1.0, threads=2)
    assert one["cores"] == 1 and two["cores"] == 2 and one["kind"] == "oracle"
    assert "2 threads" in two["sample"]
    if bench.usable_cores() >= 2:
        assert two["value"] > 1.3 * one["value"], (one, two)


def test_selection_recall():
    import numpy as np
    row = np.array([0, 1, 5, 9, 12, -1, -1], np.int32)
    assert bench.selection_recall(row, 5, [1, 9]) == 1.0
    assert bench.selection_recall(row, 5, [1, 2, 9, 40]) == 0.5
    assert bench.selection_recall(row, 3, [9]) == 0.0          # past the count
    assert bench.selection_recall(row, 5, []) == 1.0
    assert bench.parse_args([]).comparator_page == 16
    assert bench.parse_args(["--comparator-page", "0"]).comparator_page == 0


def test_scattered_page_table():
    """The paged measurement's block table: every pool page used exactly once,
    each sequence's own pages in its row, unused entries 0; lengths that are
    not multiples of the page size give no table."""
    rng = np.random.default_rng(3)
    lengths = np.array([64, 16, 0, 48])
    t = bench.scattered_page_table(lengths, 16, rng)
    assert t.dtype == np.int32 and t.shape == (4, 4)
    used = np.concatenate([t[b, :n // 16] for b, n in enumerate(lengths)])
    assert sorted(used.tolist()) == list(range(8))
    assert not t[1, 1:].any() and not t[2].any() and not t[3, 3:].any()
    assert bench.scattered_page_table(np.array([64, 20]), 16, rng) is None
    assert bench.scattered_page_table(lengths, 0, rng) is None
    big = bench.scattered_page_table(np.array([1 << 20]), 16, np.random.default_rng(1))
    assert big.shape == (1, 65536) and np.array_equal(np.sort(big[0]), np.arange(65536))


def test_split_shards_and_arguments():
    """Equal contiguous shards cover the sequence exactly; bad shard counts
    are refused."""
    for n, r in [(1 << 20, 8), (10, 3), (5, 5), (7, 1)]:
        b = bench.shard_bounds(n, r)
        assert b[0] == 0 and b[-1] == n and len(b) == r + 1
        assert all(0 <= y - x <= -(-n // r) for x, y in zip(b, b[1:]))
    assert bench.parse_args(["--split-parts", ""]).split_parts == ""
    for bad in ("0", "2,x", "65"):
        with pytest.raises(SystemExit):
            bench.parse_args(["--split-parts", bad])


def test_paged_and_split_measurements_skip_where_they_do_not_apply():
    """The paged measurement needs every length to be a multiple of the page
    size (the packed cache is then the pool); the split one shards a single
    sequence and needs its shards to exceed L2.  Both say why they skip,
    before touching a device."""
    cfg = types.SimpleNamespace(layers=2, batch=2, h_q=8, k=16, n_sink=4, n_local=8)
    wl = types.SimpleNamespace(ts=None, cfg=cfg, lengths=np.array([100, 37]), k_bytes=1 << 20, layers=[None] * 2,
                               kvs=[[None], [None]])
    r = bench.measure_paged(wl, 16, one=None)
    assert r["page_size"] == 16 and "multiple of the page size" in r["skipped"]
    r = bench.measure_split(wl, [2, 4, 8], one=None)
    assert "one sequence" in r["skipped"] and "per_parts" not in r
    wl.cfg = types.SimpleNamespace(**{**vars(cfg), "batch": 1})
    wl.lengths = np.array([4096])
    r = bench.measure_split(wl, [2, 4, 8], one=None)
    assert "fit in L2" in r["skipped"]
