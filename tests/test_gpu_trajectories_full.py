"""Selection-cache trajectories at the workloads' full sizes, through the
one-call decode step the benchmark times, against the float64 oracle.

  llama8b_b4   all 64 AR(1) decode steps of 4 sequences x 131072 tokens
  qwen7b_1m    all 16 AR(1) decode steps of layers 0, 13 and 27 at n = 1048576,
               and step 0 of every one of the 28 layers

At every step the cosine of each sequence is compared with the oracle's
(float64 on both sides), and so is the reuse decision wherever the cosine is
not within 1e-9 of theta.  A sequence that reuses must keep the previous step's
ids; a sequence that does not is scored and selected again by the oracle (votes
within 1e-3, ids exact outside the 1e-6 band and bit-exact on the GPU's own
votes), and every sequence's attention output is compared with the oracle's
attention over the same ids (2e-3).  These are the recompute-after-reuse steps:
fresh votes over the whole cache after one or more skipped steps, in a
workspace that kept a reused row in between.  Planted keys (aligned to the
first query) must all be selected at step 0.

The comparisons run on host threads while the GPU goes on to the next step.
"""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _trajectory(cfg, layer, checks, steps=None):
    """Run `steps` (default: all) decode steps of one layer with ts_decode_step;
    queue one oracle comparison per step.  Returns the reuse decisions [T, B]."""
    m = H.ts()
    li = W.layer_inputs(cfg, layer, "cuda")
    kv = m.KVCache(li.k, li.v, li.seq_offsets, cfg.h_q)
    buf = m.StepBuffers(kv, cfg.k, cfg.n_sink, cfg.n_local)
    kb, vb = W.bf16_bits(li.k), W.bf16_bits(li.v)
    T = cfg.steps if steps is None else steps
    q_prev = np.zeros((cfg.batch, cfg.h_q, cfg.head_dim), np.uint16)
    prev_ids = None
    decisions = []
    for t in range(T):
        q = li.q[t].cuda().contiguous()
        theta = cfg.theta if cfg.theta is not None else 2.0
        m.ts_decode_step(kv, q, buf.q_prev, buf.reuse, t == 0, theta, cfg.k, cfg.n_sink, cfg.n_local,
                         buf.votes, buf.ids, buf.count, buf.out, buf.ws, buf.cos)
        res = H.host_results(buf)
        qb = W.bf16_bits(q)
        for b in range(cfg.batch):
            r, c = oracle.selcache(qb[b], q_prev[b], t == 0, theta)
            assert abs(c - res["cos"][b]) < 1e-12, (layer, t, b, c, res["cos"][b])
            if abs(c - theta) > 1e-9:
                assert bool(res["reuse"][b]) == r, (layer, t, b, c)
        if t == 0:
            assert not res["reuse"].any(), "the first step never reuses"
            for b, pos in enumerate(li.planted):
                assert set(pos.tolist()) <= set(res["ids"][b].tolist()), "a planted key was not selected"
        checks.submit(H.check_arrays, kb, vb, li.seq_offsets, qb, res, cfg.k, cfg.n_sink, cfg.n_local,
                      reuse=res["reuse"].copy(), prev_ids=prev_ids)
        prev_ids = res["ids"]
        decisions.append(res["reuse"].copy())
    status, site = m.ts_get_device_status(buf.ws)
    assert status == m.TS_OK, (status, site)
    del kv, buf, li
    return np.array(decisions)


def _rate(decisions):
    """Fraction of reused (step, sequence) decisions after the first step."""
    return float(decisions[1:].mean())


def test_llama8b_b4_trajectory_full():
    cfg = W.CONFIGS["llama8b_b4"]
    checks = H.OracleChecks()
    d = _trajectory(cfg, 0, checks)
    diags = checks.join()
    rate = _rate(d)
    print("llama8b_b4 reuse rate %.3f, recomputed sequence-steps %d, worst vote rel %.3g, worst out err %.3g"
          % (rate, int((~d.astype(bool)).sum()), max(x["max_vote_rel"] for x in diags),
             max(x["max_out_err"] for x in diags)))
    # the flattened AR(1) cosine crosses 0.9 about six steps after a recompute:
    # about 57 of 64 steps reuse
    assert 0.8 < rate < 0.95, rate


@pytest.mark.parametrize("layer", [0, 13, 27])
def test_qwen7b_1m_trajectory_full(layer):
    cfg = W.CONFIGS["qwen7b_1m"]
    checks = H.OracleChecks(in_flight=8)
    d = _trajectory(cfg, layer, checks)
    diags = checks.join()
    rate = _rate(d)
    print("qwen7b_1m layer %d reuse %d of %d steps, worst vote rel %.3g, worst out err %.3g"
          % (layer, int(d[1:].sum()), cfg.steps - 1, max(x["max_vote_rel"] for x in diags),
             max(x["max_out_err"] for x in diags)))
    # about 9 or 10 of the 15 later steps reuse
    assert 0.4 < rate < 0.85, rate


def test_qwen7b_1m_step0_all_layers():
    cfg = W.CONFIGS["qwen7b_1m"]
    checks = H.OracleChecks(in_flight=6)
    for layer in range(cfg.layers):
        _trajectory(cfg, layer, checks, steps=1)
    diags = checks.join()
    assert len(diags) == cfg.layers
    print("qwen7b_1m step 0, 28 layers: worst vote rel %.3g, set diffs %d, worst out err %.3g"
          % (max(x["max_vote_rel"] for x in diags), sum(x["set_diffs"] for x in diags),
             max(x["max_out_err"] for x in diags)))
