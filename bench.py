#!/usr/bin/env python
"""Decode layer-steps/s of the TokenSelect hot path on B200 (sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole decode hot path over one batch of synthetic
input, for every layer of the workload: selection-cache decision (ts_selcache),
soft vote (ts_score), top-k + sink/local selection (ts_select) and attention
over the selected tokens (ts_sparse_attn), all through the C ABI.  The default
workload is the largest one that fits one GPU: the 1M-token decode step over
all 28 layers of a Qwen2-7B-shaped model (B=1, h_q=28, h_kv=4, d=128,
n=1048576 per layer, k=4096 + 4 sink + 1024 local, selection cache with cosine
threshold 0.9 over 16 AR(1) queries).  Every step is replayed from CUDA graphs;
inputs rotate over enough copies of the KV cache that each step reads data
that is not in L2 (at 1M tokens one step reads 28 GiB of K: no copies needed).

Two rooflines are reported.  `roofline` is the dominant kernel, score pass A
(the K scan), timed alone.  `step_roofline` is the whole step: the algorithmic
bytes of the timed steps (K of every layer-step whose selection was computed
afresh, plus the gathered K and V rows of every layer-step) over the timed
region's duration; which layer-steps reused their selection is read back from
a replay of exactly the timed sequence of steps.

Beside the main line, each measured after the timed region: `kernels` (each
kernel alone), `comparator` (the page-level comparator after Quest on the
same layers: its kernels, the per-token metadata update, recall),
`paged` (the same layers read through a scattered block table of 16-token
pages, beside the packed cache), `split` (the token-axis split of one
sequence: one rank's phases at R = 2, 4, 8, exchanges excluded) and `e2e`
(every step's queries in and outputs out through pinned host memory).

Multi-GPU (torchrun): every rank runs an independent replica of the workload
(the path has no cross-sequence exchange); the timed region is bracketed by
barriers and the elapsed time is the max over ranks.

--impl reference times the float64 CPU oracle on the same workload (rank 0
only): the pages ship no runnable implementation, so the oracle is the
reference arm.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="qwen7b_1m", choices=W.ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="run only the first N layers of the workload (a smaller case of the same kernels, "
                         "for profiler captures); the JSON line's config records it")
    ap.add_argument("--comparator-page", type=int, default=16,
                    help="page size of the page-level comparator (Quest's min/max page bounds) measured beside "
                         "the token-level path (0: not measured)")
    ap.add_argument("--paged-page", type=int, default=16,
                    help="page size of the paged-cache measurement: the same layers read through a block table "
                         "of scattered pages, timed beside the packed cache (0: not measured)")
    ap.add_argument("--split-parts", default="2,4,8",
                    help="shard counts of the token-axis split of one sequence timed on this GPU (rank 0's "
                         "phases; batch-1 workloads whose shards exceed L2; empty: not measured)")
    ap.add_argument("--eager-steps", type=int, default=None,
                    help="profiler capture mode: after set-up, run this many decode steps of the workload as "
                         "plain (not graph-replayed) C-ABI calls, along the workload's query sequence, and exit "
                         "without timing or printing a result")
    a = ap.parse_args(argv)
    big = a.workload in ("llama8b_b4", "ragged_b32", "qwen7b_1m")
    if a.steps is None:
        a.steps = {"reference": 10}.get(a.impl, 200 if big else 3000)
    if a.warmup is None:
        a.warmup = 3 if a.impl == "reference" else (10 if big else 50)
    if a.warmup < 3:
        raise SystemExit("at least 3 warm-up steps are required")
    try:
        parts = [int(x) for x in a.split_parts.split(",") if x.strip()]
    except ValueError:
        raise SystemExit("--split-parts must be a comma-separated list of shard counts")
    if any(not 1 <= r <= 64 for r in parts):
        raise SystemExit("--split-parts: shard counts must be in [1, 64]")
    if a.layers is not None and not 1 <= a.layers <= W.CONFIGS[a.workload].layers:
        raise SystemExit("--layers must be in [1, %d] for %s" % (W.CONFIGS[a.workload].layers, a.workload))
    return a


# ---------------------------------------------------------------------------
# process group
# ---------------------------------------------------------------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if torch.cuda.is_available() and self.pg.get_backend() == "nccl":
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = "cuda" if self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def aggregate(per_rank_units: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return per_rank_units * world / max_seconds


# ---------------------------------------------------------------------------
# clocks (NVML, sampled in a thread during the timed region)
# ---------------------------------------------------------------------------

_REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}
REJECT_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id, props.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # NVML missing: clocks are reported as unavailable
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in _REASON_BITS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()
        return False

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}

    def rejected(self):
        s = self.summary()
        if self.reasons & REJECT_REASONS:
            return True
        return bool(s["sm_mhz"] and s["sm_max_mhz"] and s["sm_mhz"] < 0.6 * s["sm_max_mhz"] and not self.reasons)


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "score_pass_a_traffic.json")


def profile_traffic(kernel_src: str, workload: str, path: str = TRAFFIC_RECORD):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(kernel_src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if rec.get("source_sha256") != digest:
            return None
        return rec.get("per_launch_bytes", {}).get(workload)
    except Exception:
        return None


# ---------------------------------------------------------------------------
# workload set-up
# ---------------------------------------------------------------------------

class Workload:
    def __init__(self, name: str, device, layers=None):
        import query_aware_kv_ts_b200 as ts
        self.ts = ts
        cfg = W.CONFIGS[name]
        if layers is not None:
            cfg = dataclasses.replace(cfg, layers=layers)   # range checked by parse_args
        self.cfg = cfg
        self.name = name
        self.device = device
        self.layers = []
        for layer in range(cfg.layers):
            li = W.layer_inputs(cfg, layer, device)
            self.layers.append(li)
        self.lengths = np.diff(self.layers[0].seq_offsets)
        self.k_bytes = int(self.lengths.sum()) * cfg.h_kv * cfg.head_dim * 2            # per layer
        per_step = self.k_bytes * cfg.layers
        self.rotate = max(1, math.ceil(4 * L2_BYTES / per_step)) if per_step < 4 * L2_BYTES else 1
        self.T = cfg.steps
        # rotating copies of each layer's cache (identical contents)
        self.kvs = []
        for li in self.layers:
            copies = []
            for r in range(self.rotate):
                k = li.k if r == 0 else li.k.clone()
                v = li.v if r == 0 else li.v.clone()
                copies.append(ts.KVCache(k, v, li.seq_offsets, cfg.h_q))
            self.kvs.append(copies)
        # every layer's queries in one device tensor [T, layers, B, h_q, d], so
        # that one step's inputs are one contiguous block (one host copy per
        # step end to end); q[layer] is the layer's [T, B, h_q, d] view, and
        # q[layer][t] a contiguous [B, h_q, d] query
        self.q_all = torch.stack([li.q for li in self.layers], dim=1).to(device).contiguous()
        self.q = [self.q_all[:, l] for l in range(cfg.layers)]
        self.bufs = [ts.StepBuffers(c[0], cfg.k, cfg.n_sink, cfg.n_local) for c in self.kvs]
        # and every layer's output in one [layers, B, h_q, d] tensor (one copy back)
        self.out_all = torch.zeros((cfg.layers,) + tuple(self.bufs[0].out.shape), dtype=torch.float32,
                                   device=device)
        for layer, b in enumerate(self.bufs):
            b.out = self.out_all[layer]
        self.theta = cfg.theta if cfg.theta is not None else 2.0   # 2.0: cosine never reaches it
        self.period = self.rotate * self.T // math.gcd(self.rotate, self.T)
        # device steps per replayed graph in the timed regions: a whole period
        # when steps are short (host replay overhead would otherwise show)
        self.inner = self.period if self.k_bytes * cfg.layers < 4 * L2_BYTES else 1

    def k_rows_bytes(self):
        """Algorithmic bytes of one full (non-reused) layer-step, all sequences."""
        c = self.cfg
        m = np.minimum(self.lengths, c.k + c.n_sink + c.n_local)
        return self.k_bytes + int(m.sum()) * c.h_kv * c.head_dim * 2 * 2

    # one layer-step through the public C ABI: the one-call decode step
    # (selection cache, score, select, sparse attention)
    def layer_step(self, layer: int, i: int):
        ts, b = self.ts, self.bufs[layer]
        kv = self.kvs[layer][i % self.rotate]
        q = self.q[layer][i % self.T]
        ts.ts_decode_step(kv, q, b.q_prev, b.reuse, False, self.theta, b.k, b.n_sink, b.n_local, b.votes, b.ids,
                          b.count, b.out, b.ws, b.cos)

    def step(self, i: int):
        for layer in range(self.cfg.layers):
            self.layer_step(layer, i)

    def capture(self, fn_per_index, count, inner=1):
        """count graphs; graph j replays fn_per_index(j*inner + r) for r < inner,
        so that one host-side replay covers `inner` device steps."""
        graphs = []
        for j in range(count):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for r in range(inner):
                    fn_per_index(j * inner + r)
            graphs.append(g)
        return graphs


def time_graphs(graphs, K, W_, inner=1, singles=None):
    """Seconds for exactly K device steps: K // inner replays of graphs of
    `inner` steps, then the remainder from the single-step graphs."""
    reps, rest = divmod(K, inner)
    if singles is None:
        singles, rest, reps = graphs, 0, -(-K // inner)
    for i in range(max(1, -(-W_ // inner))):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    for i in range(rest):
        singles[(reps * inner + i) % len(singles)].replay()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / 1000.0, reps * inner + rest


def replay_order(n_graphs, K, W_, inner, n_singles):
    """Step indices that time_graphs(graphs, K, W_, inner, singles) runs, in
    order: (warm-up steps, timed steps), for graphs of `inner` consecutive
    steps (graph j: steps j*inner .. j*inner + inner - 1) and single-step
    graphs (graph j: step j)."""
    reps, rest = divmod(K, inner)
    warm = [(i % n_graphs) * inner + r for i in range(max(1, -(-W_ // inner))) for r in range(inner)]
    timed = [(i % n_graphs) * inner + r for i in range(reps) for r in range(inner)]
    timed += [(reps * inner + i) % n_singles for i in range(rest)]
    return warm, timed


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------

def oracle_layer_step_fn(wl_cfg, li, max_tokens=None):
    import oracle
    off = li.seq_offsets
    kb, vb = W.bf16_bits(li.k), W.bf16_bits(li.v)
    qb = W.bf16_bits(li.q[0])
    if max_tokens is not None and off[1] > max_tokens:
        off = np.array([0, max_tokens], np.int64)
        qb = qb[:1]
    tokens = int(off[-1])

    def run():
        oracle.decode_step(kb, vb, off, qb, wl_cfg.k, wl_cfg.n_sink, wl_cfg.n_local)
    return run, tokens


def cpu_baseline(wl: Workload, budget_s: float):
    """Oracle layer-steps/s on this host, one core, on whole layer-steps of the
    workload when one fits the budget, else on a token sample of sequence 0."""
    cfg = wl.cfg
    li = wl.layers[0]
    total = int(li.seq_offsets[-1])
    run, tokens = oracle_layer_step_fn(cfg, li)
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    sample_desc = "whole %s layer-steps (%d tokens)" % (cfg.name, tokens)
    scale = 1.0
    if one > budget_s / 2:
        run, tokens = oracle_layer_step_fn(cfg, li, max_tokens=32768)
        scale = tokens / total
        sample_desc = "%d-token sample of sequence 0 of a %s layer-step, scaled by tokens" % (tokens, cfg.name)
    n, t0 = 0, time.perf_counter()
    while True:
        run()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    value = n * scale / el
    return {"value": value, "unit": "layer-steps/s", "cores": 1, "kind": "oracle",
            "sample": "%d x %s, float64 C oracle, 1 thread, %.1f s" % (n, sample_desc, el)}


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_all_cores(wl, budget_s: float, threads=None):
    """The same oracle on every usable core: independent layer-steps on as many
    threads (the oracle's C calls release the interpreter lock, so the threads
    run in parallel); the oracle itself is unchanged."""
    cfg = wl.cfg
    li = wl.layers[0]
    total = int(li.seq_offsets[-1])
    run, tokens = oracle_layer_step_fn(cfg, li)
    scale = 1.0
    sample_desc = "whole %s layer-steps (%d tokens)" % (cfg.name, tokens)
    t0 = time.perf_counter()
    run()
    if time.perf_counter() - t0 > budget_s / 4:
        run, tokens = oracle_layer_step_fn(cfg, li, max_tokens=32768)
        scale = tokens / total
        sample_desc = "%d-token samples of sequence 0 of %s layer-steps, scaled by tokens" % (tokens, cfg.name)
    n_threads = threads or usable_cores()
    counts = [0] * n_threads
    stop_at = time.perf_counter() + budget_s

    def worker(i):
        while time.perf_counter() < stop_at:
            run()
            counts[i] += 1
    t0 = time.perf_counter()
    pool = [threading.Thread(target=worker, args=(i,)) for i in range(n_threads)]
    for t in pool:
        t.start()
    for t in pool:
        t.join()
    el = time.perf_counter() - t0
    n = sum(counts)
    return {"value": n * scale / el, "unit": "layer-steps/s", "cores": n_threads, "kind": "oracle",
            "sample": "%d x %s, float64 C oracle, %d threads, %.1f s" % (n, sample_desc, n_threads, el)}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def selection_recall(ids: np.ndarray, count: int, want) -> float:
    """Fraction of the token ids `want` that the selected row ids[:count] holds
    (1.0 when `want` is empty)."""
    want = set(int(x) for x in want)
    if not want:
        return 1.0
    return len(want & set(ids[:count].tolist())) / len(want)


def measure_comparator(wl, P: int, one, peak: float, peak_kind: str) -> dict:
    """The page-level comparator (Quest's min/max page bounds, pages of P
    tokens) on the same layers, queries and selection budget as the
    token-level path: per-layer times of its kernels alone (the full metadata
    pass, and the update of the newest token's page that a decode loop runs
    per token, apart), the score kernel's
    bandwidth, and on layer 0 how many planted query-aligned keys each method
    selects and how much of the token-level selection the page selection
    covers."""
    ts, cfg = wl.ts, wl.cfg
    qb = [[ts.QuestBuffers(kv, P) for kv in copies] for copies in wl.kvs]
    ids = [torch.full_like(b.ids, -1) for b in wl.bufs]
    count = [torch.zeros_like(b.count) for b in wl.bufs]
    out = [torch.zeros_like(b.out) for b in wl.bufs]

    def kv_of(l, i):
        return wl.kvs[l][i % wl.rotate], qb[l][i % wl.rotate]

    for l in range(cfg.layers):
        for r in range(wl.rotate):
            ts.ts_quest_metadata(wl.kvs[l][r], P, qb[l][r].kmin, qb[l][r].kmax)

    def score(l, i):
        kv, b = kv_of(l, i)
        ts.ts_quest_score(kv, wl.q[l][i % wl.T], P, b.kmin, b.kmax, b.scores)

    def select(l, i):
        kv, b = kv_of(l, i)
        ts.ts_quest_select(kv, b.scores, P, cfg.k, cfg.n_sink, cfg.n_local, ids[l], count[l])

    def attn(l, i):
        ts.ts_sparse_attn(wl.kvs[l][i % wl.rotate], wl.q[l][i % wl.T], ids[l], count[l], out[l], wl.bufs[l].ws)

    res = {"method": "page-level min/max key bounds (Quest), head-summed, top floor(k/P) pages + the windows",
           "page_size": P}
    res["metadata_us"] = 1e6 * one(lambda i: [ts.ts_quest_metadata(kv_of(l, i)[0], P, kv_of(l, i)[1].kmin,
                                                                    kv_of(l, i)[1].kmax)
                                              for l in range(cfg.layers)])
    # a decode loop's per-token cost: the page that took the newest token
    res["metadata_update_us"] = 1e6 * one(
        lambda i: [ts.ts_quest_metadata_update(kv_of(l, i)[0], P, 1, kv_of(l, i)[1].kmin, kv_of(l, i)[1].kmax)
                   for l in range(cfg.layers)])
    res["score_us"] = 1e6 * one(lambda i: [score(l, i) for l in range(cfg.layers)])
    res["select_us"] = 1e6 * one(lambda i: [select(l, i) for l in range(cfg.layers)])
    res["sparse_attn_us"] = 1e6 * one(lambda i: [attn(l, i) for l in range(cfg.layers)])
    res["step_us"] = 1e6 * one(lambda i: [(score(l, i), select(l, i), attn(l, i)) for l in range(cfg.layers)])
    pages = int(sum(-(-int(n) // P) for n in wl.lengths))
    score_bytes = 2 * pages * cfg.h_kv * cfg.head_dim * 2
    res["score_roofline"] = {"bound": "hbm", "alg_bytes_per_launch": score_bytes,
                             "achieved": score_bytes / (res["score_us"] * 1e-6) / 1e9, "peak": peak,
                             "peak_kind": peak_kind, "unit": "GB/s"}
    res["score_roofline"]["frac"] = res["score_roofline"]["achieved"] / peak
    # recall on layer 0, first query, every sequence: both methods select afresh
    b0 = wl.bufs[0]
    kv0, q0 = wl.kvs[0][0], wl.q[0][0]
    ts.ts_score(kv0, q0, None, b0.votes, b0.ws)
    ts.ts_select(kv0, b0.votes, cfg.k, cfg.n_sink, cfg.n_local, None, b0.ids, b0.count, b0.ws)
    score(0, 0)
    select(0, 0)
    torch.cuda.synchronize()
    t_ids, t_cnt = b0.ids.cpu().numpy(), b0.count.cpu().numpy()
    p_ids, p_cnt = ids[0].cpu().numpy(), count[0].cpu().numpy()
    planted = wl.layers[0].planted
    rec_p, rec_t, cover = [], [], []
    for bb in range(cfg.batch):
        if planted is not None and len(planted[bb]):
            rec_p.append(selection_recall(p_ids[bb], int(p_cnt[bb]), planted[bb]))
            rec_t.append(selection_recall(t_ids[bb], int(t_cnt[bb]), planted[bb]))
        cover.append(selection_recall(p_ids[bb], int(p_cnt[bb]), t_ids[bb][:int(t_cnt[bb])]))
    res["planted_recall"] = float(np.mean(rec_p)) if rec_p else None
    res["tokenselect_planted_recall"] = float(np.mean(rec_t)) if rec_t else None
    res["covers_tokenselect_selection"] = float(np.mean(cover))
    del qb
    return res


def scattered_page_table(lengths, P: int, rng):
    """Block table of a pool that holds exactly the sequences' pages of P
    tokens, each sequence's pages at distinct pool pages drawn as one random
    permutation of the pool: int32 [B, max pages], unused entries 0.  None
    when a length is not a multiple of P (the pool is then not the packed
    cache)."""
    lengths = np.asarray(lengths, np.int64)
    if P <= 0 or np.any(lengths % P):
        return None
    pages = lengths // P
    perm = rng.permutation(int(pages.sum())).astype(np.int32)
    table = np.zeros((lengths.size, max(1, int(pages.max()))), np.int32)
    o = 0
    for b, c in enumerate(pages):
        table[b, :c] = perm[o:o + c]
        o += c
    return table


def measure_paged(wl, P: int, one) -> dict:
    """The same layers as a paged cache (pages of P tokens): the packed K and
    V tensors serve as the pool and each layer's block table scatters every
    sequence's pages over it at random, as in a serving pool, so no copy is
    made (the paged sequence is the packed one with its pages permuted, the
    same amount of work).  Timed beside the packed cache, every layer-step
    scored afresh (the selection cache off) on both: the scoring scan alone,
    the whole one-call step, and the attention gather alone."""
    ts, cfg = wl.ts, wl.cfg
    res = {"page_size": P, "table": "one random permutation of the pool's pages per layer (seeded)"}
    rng = np.random.default_rng(20240)
    pkvs = []
    for l in range(cfg.layers):
        table = scattered_page_table(wl.lengths, P, rng)
        if table is None:
            res["skipped"] = "a sequence length is not a multiple of the page size"
            return res
        t = torch.from_numpy(table).to(wl.device)
        pkvs.append([ts.KVCache(c.k, c.v, wl.layers[l].seq_offsets, cfg.h_q, page_table=t, page_size=P)
                     for c in wl.kvs[l]])
    kvs = {"packed": wl.kvs, "paged": pkvs}
    bufs = {"packed": wl.bufs, "paged": [ts.StepBuffers(c[0], cfg.k, cfg.n_sink, cfg.n_local) for c in pkvs]}

    def fresh_step(name, l, i):
        b = bufs[name][l]
        ts.ts_decode_step(kvs[name][l][i % wl.rotate], wl.q[l][i % wl.T], b.q_prev, b.reuse, True, 2.0, b.k,
                          b.n_sink, b.n_local, b.votes, b.ids, b.count, b.out, b.ws, b.cos)

    for name in kvs:                 # eager first calls (kernel attributes, tensor maps) before any capture
        for l in range(cfg.layers):
            fresh_step(name, l, 0)
    torch.cuda.synchronize()
    for key in ("score_pass_a_us", "step_us", "sparse_attn_us"):
        res[key] = {}
    for name in kvs:
        kv_, bf = kvs[name], bufs[name]
        res["score_pass_a_us"][name] = 1e6 * one(
            lambda i: [ts.ts_score_logits(kv_[l][i % wl.rotate], wl.q[l][i % wl.T], None, bf[l].ws)
                       for l in range(cfg.layers)])
        res["step_us"][name] = 1e6 * one(lambda i: [fresh_step(name, l, i) for l in range(cfg.layers)])
        res["sparse_attn_us"][name] = 1e6 * one(
            lambda i: [ts.ts_sparse_attn(kv_[l][i % wl.rotate], wl.q[l][i % wl.T], bf[l].ids, bf[l].count,
                                         bf[l].out, bf[l].ws) for l in range(cfg.layers)])
    del bufs["paged"]
    return res


def shard_bounds(n: int, parts: int):
    """Equal contiguous shards of n tokens over `parts` ranks: [t_r, t_{r+1})."""
    return [n * r // parts for r in range(parts + 1)]


def measure_split(wl, parts_list, one) -> dict:
    """The token-axis split of one sequence (query_aware_kv_ts_b200.split) on
    this GPU: every layer's sequence cut into R equal shards (views of the
    packed cache), one emulated step run to fill every shard's gathered
    buffers (all shards' phases, the all-gathers as copies), then rank 0's
    phases alone timed over the layers, in total and phase by phase: one
    rank's compute per layer-step, the three all-gathers not included."""
    from query_aware_kv_ts_b200 import split
    ts, cfg = wl.ts, wl.cfg
    res = {"what": "rank 0's phases per layer-step, exchanges excluded; equal shards; each phase alone and "
                   "all five in order",
           "phases": ["normalisers (pass A + merge)", "votes (normaliser join + pass B)",
                      "candidates (shard selection + keys)", "select_and_attend (key merge + attention with lse)",
                      "join (attention merge)"]}
    if cfg.batch != 1:
        res["skipped"] = "the split shards one sequence (batch 1)"
        return res
    if wl.k_bytes * cfg.layers // max(parts_list) < 4 * L2_BYTES:
        res["skipped"] = "one rank's shards of all layers fit in L2 at the largest shard count"
        return res
    n = int(wl.lengths[0])
    res["per_parts"] = {}
    for R in parts_list:
        bounds = shard_bounds(n, R)
        shards = []
        for l in range(cfg.layers):
            kv = wl.kvs[l][0]
            row = []
            for r in range(R):
                t0, t1 = bounds[r], bounds[r + 1]
                skv = ts.KVCache(kv.k[t0:t1], kv.v[t0:t1], np.array([0, t1 - t0]), cfg.h_q)
                row.append((skv, split.ShardBuffers(skv, cfg.k, cfg.n_sink, cfg.n_local, R), t0))
            shards.append(row)
        for l in range(cfg.layers):
            split.emulate_split_decode_step(shards[l], wl.q[l][0], n)
        torch.cuda.synchronize()

        def phase(name, l):
            kv, b, t = shards[l][0]
            q = wl.q[l][0]
            if name == "normalisers":
                split.phase_normalisers(kv, q, b)
            elif name == "votes":
                split.phase_votes(kv, b)
            elif name == "candidates":
                split.phase_candidates(kv, b, t, n)
            elif name == "select_and_attend":
                split.phase_select_and_attend(kv, q, b, 0, t, n)
            else:
                split.phase_join_attention(b)

        names = ["normalisers", "votes", "candidates", "select_and_attend", "join"]
        per = {"shard_tokens": bounds[1] - bounds[0], "phases_us": {}}
        for name in names:
            per["phases_us"][name] = 1e6 * one(lambda i: [phase(name, l) for l in range(cfg.layers)])
        per["rank_compute_us"] = 1e6 * one(lambda i: [phase(nm, l) for l in range(cfg.layers) for nm in names])
        res["per_parts"][str(R)] = per
        del shards
    return res


def run_ours(a, d: Dist):
    torch.cuda.set_device(d.local)
    dev = torch.device("cuda", d.local)
    d.init("nccl")
    wl = Workload(a.workload, dev, a.layers)
    cfg = wl.cfg
    ts = wl.ts
    if a.eager_steps is not None:
        for i in range(a.eager_steps):
            wl.step(i)
        torch.cuda.synchronize()
        d.close()
        return

    # eager warm-up (also configures kernel attributes before capture)
    for i in range(2):
        wl.step(i)
    torch.cuda.synchronize()
    # one graph per step of the query / rotation period (the end-to-end loop
    # replays these), and graphs of `inner` consecutive steps for the device
    # timing, so that host-side replay overhead is not in the device numbers
    graphs = wl.capture(wl.step, wl.period)
    inner = wl.inner
    graphs_n = wl.capture(wl.step, max(1, wl.period // inner), inner)

    # ---- main timed region: whole steps ----
    # every layer starts from an empty selection-cache state (first step
    # recomputes), as the record pass below does
    for b in wl.bufs:
        b.q_prev.zero_()
    d.barrier()
    torch.cuda.synchronize()
    for attempt in range(2):
        if attempt:
            for b in wl.bufs:
                b.q_prev.zero_()
        with ClockSampler(d.local) as clk:
            el, steps_run = time_graphs(graphs_n, a.steps, a.warmup, inner, graphs)
        if not clk.rejected():
            break
    d.barrier()
    el_max = d.max(el)
    layer_steps = steps_run * cfg.layers
    value = aggregate(layer_steps, d.world, el_max)
    ms_per_step = el_max / steps_run * 1000.0

    # ---- dominant kernel alone: score pass A (ts_score_logits: the K scan,
    #      every sequence scored) ----
    Ka = max(a.steps, 20)

    def one(fn):
        g = wl.capture(fn, 1, wl.rotate)
        el_k, k_run = time_graphs(g, Ka, a.warmup, wl.rotate)
        return el_k / (k_run * cfg.layers)
    per_launch_s = one(lambda i: [ts.ts_score_logits(wl.kvs[l][i % wl.rotate], wl.q[l][i % wl.T], None,
                                                     wl.bufs[l].ws) for l in range(cfg.layers)])
    peak, peak_kind = measured_hbm_peak()
    achieved = wl.k_bytes / per_launch_s / 1e9
    traffic = profile_traffic(os.path.join(ROOT, "query_aware_kv_ts_b200", "csrc", "score.cu"), a.workload)

    # per-kernel breakdown (each kernel alone, same rotation), with the fused
    # one-kernel scoring beside the two passes
    kernels = {"score_pass_a_us": per_launch_s * 1e6}
    kernels["score_pass_b_us"] = 1e6 * one(
        lambda i: [ts.ts_score_vote(wl.kvs[l][i % wl.rotate], None, wl.bufs[l].votes, wl.bufs[l].ws)
                   for l in range(cfg.layers)])
    kernels["score_fused_us"] = 1e6 * one(
        lambda i: [ts.ts_score_fused(wl.kvs[l][i % wl.rotate], wl.q[l][i % wl.T], None, wl.bufs[l].votes,
                                     wl.bufs[l].ws) for l in range(cfg.layers)])
    kernels["select_us"] = 1e6 * one(lambda i: [ts.ts_select(wl.kvs[l][i % wl.rotate], wl.bufs[l].votes, cfg.k,
                                                             cfg.n_sink, cfg.n_local, None, wl.bufs[l].ids,
                                                             wl.bufs[l].count, wl.bufs[l].ws)
                                                for l in range(cfg.layers)])
    kernels["sparse_attn_us"] = 1e6 * one(lambda i: [ts.ts_sparse_attn(wl.kvs[l][i % wl.rotate], wl.q[l][i % wl.T],
                                                                       wl.bufs[l].ids, wl.bufs[l].count,
                                                                       wl.bufs[l].out, wl.bufs[l].ws)
                                                     for l in range(cfg.layers)])
    # the same attention with its dot products on the CUDA cores (fp32 FMA)
    # instead of the tensor cores, for the comparison
    os.environ["TS_ATTN_CUDA_CORES"] = "1"
    try:
        kernels["sparse_attn_cuda_cores_us"] = 1e6 * one(
            lambda i: [ts.ts_sparse_attn(wl.kvs[l][i % wl.rotate], wl.q[l][i % wl.T], wl.bufs[l].ids,
                                         wl.bufs[l].count, wl.bufs[l].out, wl.bufs[l].ws)
                       for l in range(cfg.layers)])
    finally:
        del os.environ["TS_ATTN_CUDA_CORES"]

    comparator = None
    if a.comparator_page:
        comparator = measure_comparator(wl, a.comparator_page, one, peak, peak_kind)

    paged = measure_paged(wl, a.paged_page, one) if a.paged_page else None
    split_parts = [int(x) for x in a.split_parts.split(",") if x.strip()]
    split_res = measure_split(wl, split_parts, one) if split_parts else None
    if split_res is not None and paged is not None and "step_us" in paged:
        split_res["one_gpu_fresh_step_us"] = paged["step_us"]["packed"]

    # ---- end to end: pinned host query in, result out, every step ----
    # one step's inputs: every layer's query of that step, one contiguous
    # block; its result: every layer's output, one contiguous block
    q_host = wl.q_all.cpu().pin_memory()
    out_host = torch.empty_like(wl.out_all, device="cpu").pin_memory()
    h2d = q_host[0].numel() * q_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    K_e2e = min(a.steps, 2000)

    def e2e_step(i):
        wl.q_all[i % wl.T].copy_(q_host[i % wl.T], non_blocking=True)
        graphs[i % len(graphs)].replay()
        out_host.copy_(wl.out_all, non_blocking=True)
        torch.cuda.synchronize()
    for i in range(a.warmup):
        e2e_step(i)
    d.barrier()
    t0 = time.perf_counter()
    for i in range(K_e2e):
        e2e_step(i)
    e2e_el = d.max(time.perf_counter() - t0)
    e2e_value = aggregate(K_e2e * cfg.layers, d.world, e2e_el)

    # which layer-steps of the timed region reused their selection: replay the
    # same sequence of steps from the same empty state with single-step graphs
    # and read every layer's reuse flags after each timed step
    warm_idx, timed_idx = replay_order(len(graphs_n), steps_run, a.warmup, inner, len(graphs))
    assert len(timed_idx) == steps_run
    flags = torch.zeros((steps_run, cfg.layers, cfg.batch), dtype=torch.int32, device=dev)
    for b in wl.bufs:
        b.q_prev.zero_()
    for j in warm_idx:
        graphs[j % len(graphs)].replay()
    for t, j in enumerate(timed_idx):
        graphs[j % len(graphs)].replay()
        for layer in range(cfg.layers):
            flags[t, layer].copy_(wl.bufs[layer].reuse)
    torch.cuda.synchronize()
    flags_np = flags.cpu().numpy().astype(bool)
    reuse_rate = float(flags_np.mean()) if cfg.theta is not None else None
    # algorithmic bytes of the timed steps: K of each (layer-step, sequence)
    # scored afresh, gathered K and V rows of every one
    row_bytes = cfg.h_kv * cfg.head_dim * 2
    m_b = np.minimum(wl.lengths, cfg.k + cfg.n_sink + cfg.n_local)
    k_part = int(((~flags_np) * (wl.lengths * row_bytes)[None, None, :]).sum())
    gather_part = int(m_b.sum()) * row_bytes * 2 * cfg.layers * steps_run
    step_alg_bytes = k_part + gather_part
    step_hbm_gbs = step_alg_bytes / el_max / 1e9

    # every layer-step is one ts_decode_step call (the same shapes in every
    # layer); with TS_REUSE_SKIP=1 a graph-replayed layer-step in which every
    # sequence reuses its selection skips the scoring and selection kernels
    # (the cosine test and the two attention kernels run)
    kernels_per_layer_step = ts.ts_decode_step_kernels(wl.kvs[0][0], cfg.k, cfg.n_sink, cfg.n_local)
    skip_on = cfg.theta is not None and os.environ.get("TS_REUSE_SKIP") == "1"
    all_reused = flags_np.all(axis=2) if skip_on else np.zeros(flags_np.shape[:2], bool)
    gpu_launches = int(np.where(all_reused, 3, kernels_per_layer_step).sum())
    alg_bytes = wl.k_rows_bytes() * cfg.layers
    result = {
        "metric": "decode layer-steps/s (score+select+sparse-attn); HBM GB/s vs roofline",
        "value": value,
        "unit": "layer-steps/s",
        "n_gpus": d.world,
        "steps": steps_run,
        "warmup": a.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": a.workload, "batch": cfg.batch, "h_q": cfg.h_q, "h_kv": cfg.h_kv,
                   "head_dim": cfg.head_dim, "n": int(wl.lengths.max()), "tokens_total": int(wl.lengths.sum()),
                   "layers": cfg.layers, "k": cfg.k, "n_sink": cfg.n_sink, "n_local": cfg.n_local,
                   "selection_cache_theta": cfg.theta, "parallelism": "replicas" if d.world > 1 else "single",
                   "l2": "inputs larger than L2: %d rotating KV copies, %.0f MiB of K read per rotation"
                         % (wl.rotate, wl.rotate * wl.k_bytes * cfg.layers / 2**20),
                   "graphs": "C-ABI calls captured in CUDA graphs of %d consecutive steps" % inner},
        "step_hbm_gbs": step_hbm_gbs,
        "step_alg_bytes": step_alg_bytes / steps_run,
        "step_roofline": {"bound": "hbm", "scope": "whole decode step (all layers): K of the layer-steps "
                          "scored afresh + gathered K/V rows of every layer-step, over the timed region",
                          "achieved": step_hbm_gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                          "frac": step_hbm_gbs / peak, "alg_bytes_per_step": step_alg_bytes / steps_run,
                          "alg_bytes_no_reuse_per_step": alg_bytes,
                          "k_scored_fraction": float((~flags_np).mean())},
        "roofline": {"bound": "hbm", "kernel": "score pass A (ts_score_logits)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "alg_bytes_per_launch": wl.k_bytes,
                     "launch_us": per_launch_s * 1e6},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": "layer-steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "every step: the step's queries of all layers copied in from pinned host memory (one "
                       "copy), the graph of the C-ABI calls replayed, the fp32 outputs of all layers copied "
                       "out (one copy) and synchronised; host wall clock"},
        "gpu_launches": gpu_launches,
        "clocks": clk.summary(),
    }
    if reuse_rate is not None:
        result["reuse_rate"] = reuse_rate
    if comparator is not None:
        comparator["tokenselect_layer_step_us"] = ms_per_step * 1000.0 / cfg.layers
        result["comparator"] = comparator
    if paged is not None:
        result["paged"] = paged
    if split_res is not None:
        result["split"] = split_res
    if d.world == 1 and not a.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, a.cpu_seconds)
        result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(wl, 4.0)
    del graphs, graphs_n
    d.close()
    if d.rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(a, d: Dist):
    """The float64 oracle as the reference arm: rank 0 times it on the host."""
    if d.rank != 0:
        return
    cfg = W.CONFIGS[a.workload]
    li = W.layer_inputs(cfg, 0, "cpu")
    total = int(li.seq_offsets[-1])
    lengths = np.diff(li.seq_offsets)
    run, tokens = oracle_layer_step_fn(cfg, li)
    scale = 1.0
    sample = "one whole %s layer-step (%d tokens) per step" % (cfg.name, tokens)
    t0 = time.perf_counter()
    run()
    if time.perf_counter() - t0 > 2.0:
        run, tokens = oracle_layer_step_fn(cfg, li, max_tokens=32768)
        scale = tokens / total
        sample = "%d-token sample of sequence 0 of a %s layer-step per step, scaled by tokens" % (tokens, cfg.name)
    for _ in range(a.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        run()
    el = time.perf_counter() - t0
    value = a.steps * scale / el
    res = {"impl": "reference", "metric": "decode layer-steps/s (score+select+sparse-attn); HBM GB/s vs roofline",
           "value": value, "unit": "layer-steps/s", "n_gpus": d.world, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": el / a.steps * 1000.0, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": a.workload, "batch": cfg.batch, "h_q": cfg.h_q, "h_kv": cfg.h_kv,
                      "head_dim": cfg.head_dim, "n": int(lengths.max()), "tokens_total": total,
                      "layers": cfg.layers, "k": cfg.k, "n_sink": cfg.n_sink, "n_local": cfg.n_local,
                      "selection_cache_theta": cfg.theta, "parallelism": "host, one thread (rank 0)"},
           "cpu_baseline": {"value": value, "unit": "layer-steps/s", "cores": 1, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "layer-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(res), flush=True)


def main(argv=None):
    a = parse_args(argv)
    d = Dist()
    if a.impl == "reference":
        run_reference(a, d)
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    run_ours(a, d)
    return 0


if __name__ == "__main__":
    sys.exit(main())
