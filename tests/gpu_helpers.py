"""Helpers of the GPU parity tests: run one decode layer-step through the C ABI
(query_aware_kv_ts_b200) and compare it with the float64 oracle.

Tolerances (TokenSelect decode-step parity contract):
  votes    |v_gpu - v_ref| <= 1e-3 * v_ref + 1e-30      (relative; absolute floor
                                                          for fp32-underflowed votes)
  ids      exact, except tokens whose oracle vote lies within 1e-6 relative of
           the oracle's k-th candidate vote
  ids      bit-exact against the oracle's selection run on the GPU's own fp32
           votes (the integer decision taken in the kernel's precision)
  out      max |out_gpu - out_ref| <= 2e-3, out_ref = oracle attention over the
           same ids
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
import workloads as W

VOTE_RTOL = 1e-3
VOTE_ATOL = 1e-30
SET_BAND = 1e-6
OUT_ATOL = 2e-3


def ts():
    import query_aware_kv_ts_b200 as m
    return m


class Case:
    """Inputs of one layer-step on the device plus their host bf16 bits."""

    def __init__(self, k, v, seq_offsets, q, *, scale=0.0):
        self.k, self.v = k, v
        self.off = np.asarray(seq_offsets, np.int64)
        self.q = q.contiguous()                  # [B, h_q, d] bf16, device
        self.B = self.off.size - 1
        self.h_q = q.shape[1]
        self.scale = scale
        self.kv = ts().KVCache(k, v, self.off, self.h_q, scale)
        self.kb = W.bf16_bits(k)
        self.vb = W.bf16_bits(v)

    def oracle_scale(self):
        return None if self.scale == 0.0 else float(np.float32(self.scale))

    def seq(self, b):
        return int(self.off[b]), int(self.off[b + 1])


def run_step(case: Case, k, n_sink, n_local, buf=None, *, theta=None, first_step=True,
             reuse_override=None):
    """selcache (optional) -> score -> select -> sparse attention on the GPU."""
    m = ts()
    if buf is None:
        buf = m.StepBuffers(case.kv, k, n_sink, n_local)
    reuse = None
    if theta is not None:
        m.ts_selcache(case.q, buf.q_prev, buf.reuse, first_step, theta, buf.cos)
        reuse = buf.reuse
    if reuse_override is not None:
        buf.reuse.copy_(torch.as_tensor(np.asarray(reuse_override, np.int32)))
        reuse = buf.reuse
    m.ts_score(case.kv, case.q, reuse, buf.votes, buf.ws)
    m.ts_select(case.kv, buf.votes, k, n_sink, n_local, reuse, buf.ids, buf.count, buf.ws)
    m.ts_sparse_attn(case.kv, case.q, buf.ids, buf.count, buf.out, buf.ws)
    torch.cuda.synchronize()
    return buf


def check_votes(v_gpu: np.ndarray, v_ref: np.ndarray, h_q: int):
    err = np.abs(v_gpu.astype(np.float64) - v_ref)
    bad = err > VOTE_RTOL * v_ref + VOTE_ATOL
    assert not bad.any(), "votes: %d entries off, worst rel %.3g" % (
        bad.sum(), (err / np.maximum(v_ref, 1e-300)).max())
    if v_ref.size:
        assert abs(v_gpu.astype(np.float64).sum() - h_q) < 1e-4 * h_q
    return float((err / np.maximum(v_ref, 1e-300)).max()) if v_ref.size else 0.0


def band_mask(v_ref: np.ndarray, n: int, k: int, n_sink: int, n_local: int):
    """Tokens whose oracle vote lies within SET_BAND of the k-th candidate vote."""
    s_end, l0 = oracle.windows(n, n_sink, n_local)
    cand = np.arange(s_end, l0)
    mask = np.zeros(n, bool)
    if k <= 0 or cand.size <= k:
        return mask
    order = cand[np.lexsort((cand, -v_ref[cand]))]
    vk = v_ref[order[k - 1]]
    mask[cand] = np.abs(v_ref[cand] - vk) <= SET_BAND * vk
    return mask


def check_ids(ids_gpu, count_gpu, ids_ref, count_ref, v_ref, n, k, n_sink, n_local):
    a = set(ids_gpu[:count_gpu].tolist())
    b = set(ids_ref[:count_ref].tolist())
    assert count_gpu == count_ref, (count_gpu, count_ref)
    assert np.all(np.diff(ids_gpu[:count_gpu]) > 0), "ids not ascending"
    assert (ids_gpu[count_gpu:] == -1).all(), "padding must be -1"
    diff = a ^ b
    if diff:
        band = band_mask(v_ref, n, k, n_sink, n_local)
        outside = [i for i in diff if not band[i]]
        assert not outside, "selection differs outside the 1e-6 band: %s" % outside[:10]
    return len(diff)


def check_select_same_precision(v_gpu: np.ndarray, ids_gpu, count_gpu, k, n_sink, n_local):
    """The selection decision taken on the GPU's own fp32 votes is exact."""
    want, m = oracle.select(v_gpu.astype(np.float64), k, n_sink, n_local)
    assert count_gpu == m, (count_gpu, m)
    assert np.array_equal(ids_gpu, want), "select differs from the oracle on identical votes"


def host_results(buf) -> dict:
    """Host copies of one layer-step's results (votes, ids, count, out, reuse,
    cos), taken right after the step so the device buffers can be reused."""
    return {n: getattr(buf, n).cpu().numpy().copy() for n in ("votes", "ids", "count", "out", "reuse", "cos")}


def check_arrays(kb, vb, off, qb, res: dict, k, n_sink, n_local, *, scale=None, reuse=None, prev_ids=None):
    """Compare one layer-step's host results with the oracle, sequence by
    sequence.  kb, vb: uint16 [sum_n, h_kv, d]; off: int64 [B+1]; qb: uint16
    [B, h_q, d]; res: host_results().  A sequence with reuse[b] set must have
    kept prev_ids[b]; any other is scored and selected again by the oracle.
    Returns a dict of diagnostics (max vote error, set differences)."""
    votes, ids, count, out = res["votes"], res["ids"], res["count"], res["out"]
    h_q = qb.shape[1]
    diag = {"max_vote_rel": 0.0, "set_diffs": 0, "max_out_err": 0.0}
    for b in range(off.size - 1):
        lo, hi = int(off[b]), int(off[b + 1])
        n = hi - lo
        kbb, vbb = kb[lo:hi], vb[lo:hi]
        if reuse is not None and reuse[b]:
            assert np.array_equal(ids[b], prev_ids[b]), "reused sequence changed its ids"
        else:
            v_ref, _ = oracle.votes(kbb, qb[b], scale)
            rel = check_votes(votes[lo:hi], v_ref, h_q)
            diag["max_vote_rel"] = max(diag["max_vote_rel"], rel)
            ids_ref, m_ref = oracle.select(v_ref, k, n_sink, n_local)
            diag["set_diffs"] += check_ids(ids[b], int(count[b]), ids_ref, m_ref, v_ref, n, k, n_sink, n_local)
            check_select_same_precision(votes[lo:hi], ids[b], int(count[b]), k, n_sink, n_local)
        m_b = int(count[b])
        o_ref = oracle.sparse_attn(kbb, vbb, qb[b], ids[b], m_b, scale)
        err = float(np.abs(out[b] - o_ref).max()) if o_ref.size else 0.0
        assert err <= OUT_ATOL, "attention output off by %.3g (sequence %d)" % (err, b)
        diag["max_out_err"] = max(diag["max_out_err"], err)
    return diag


def check_step(case: Case, buf, k, n_sink, n_local, *, reuse=None, prev_ids=None, ref=None):
    """Compare one GPU layer-step with the oracle, sequence by sequence.
    Returns a dict of diagnostics (max vote error, set differences)."""
    return check_arrays(case.kb, case.vb, case.off, W.bf16_bits(case.q), host_results(buf), k, n_sink, n_local,
                        scale=case.oracle_scale(), reuse=reuse, prev_ids=prev_ids)


class OracleChecks:
    """Oracle comparisons run on host threads while the GPU goes on (the
    oracle's C calls release the interpreter lock).  At most `in_flight`
    checks are queued at once, which bounds the host memory their inputs hold.
    join() waits for all of them and re-raises the first failure."""

    def __init__(self, in_flight: int | None = None):
        import concurrent.futures as cf
        import threading
        try:
            cores = len(os.sched_getaffinity(0))
        except AttributeError:
            cores = os.cpu_count() or 1
        self.workers = max(1, cores)
        self._pool = cf.ThreadPoolExecutor(max_workers=self.workers)
        self._slots = threading.BoundedSemaphore(in_flight or 2 * self.workers)
        self._futures = []

    def submit(self, fn, *args, **kw):
        self._slots.acquire()

        def run():
            try:
                return fn(*args, **kw)
            finally:
                self._slots.release()
        self._futures.append(self._pool.submit(run))

    def join(self) -> list:
        try:
            return [f.result() for f in self._futures]
        finally:
            self._pool.shutdown(wait=True)


def config_case(cfg: W.Config, layer=0, step=0, n_override=None, device="cuda"):
    li = W.layer_inputs(cfg, layer, device, n_override=n_override)
    q = li.q[step].to(device)
    return Case(li.k, li.v, li.seq_offsets, q), li
