"""ts_decode_step captured into CUDA graphs with the selection cache on and
TS_REUSE_SKIP=1: the scoring and selection kernels sit in a conditional node
that the cosine kernel switches off when every sequence of the step reuses
its selection.
Replaying the captured steps must give, at every step of an AR(1) query
trajectory, exactly (bit for bit) what the eager one-call step gives, and the
graph-replayed trajectory must follow the oracle."""
import numpy as np
import pytest
import torch

import gpu_helpers as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _step(m, case, buf, cfg, t, stream=None):
    m.ts_decode_step(case.kv, case.q, buf.q_prev, buf.reuse, t == 0, cfg.theta, cfg.k, cfg.n_sink, cfg.n_local,
                     buf.votes, buf.ids, buf.count, buf.out, buf.ws, buf.cos, stream)


@pytest.mark.parametrize("cfg_name,n", [("llama8b_b4", 4096), ("qwen7b_1m", 16384), ("qwen7b_32k_theta", 32768)])
def test_graph_replay_equals_eager_trajectory(cfg_name, n, monkeypatch):
    monkeypatch.setenv("TS_REUSE_SKIP", "1")
    if cfg_name == "qwen7b_32k_theta":
        # the Qwen2-7B layer with the selection cache on and AR(1) queries
        import dataclasses
        cfg = dataclasses.replace(W.CONFIGS["qwen7b_32k"], steps=12, theta=0.9, ar_rho=0.95)
    else:
        cfg = W.CONFIGS[cfg_name]
    case, li = H.config_case(cfg, n_override=n)
    m = H.ts()
    be = m.StepBuffers(case.kv, cfg.k, cfg.n_sink, cfg.n_local)
    bg = m.StepBuffers(case.kv, cfg.k, cfg.n_sink, cfg.n_local)
    q_static = li.q[0].cuda().contiguous()
    gcase = H.Case(case.k, case.v, case.off, q_static)
    stream = torch.cuda.Stream()
    # one captured step, replayed for every later step (the query is copied
    # into the captured input between replays)
    graph = None
    q_prev = np.zeros((cfg.batch, cfg.h_q, cfg.head_dim), np.uint16)
    prev_ids = None
    all_reused = 0
    for t in range(cfg.steps):
        case.q = li.q[t].cuda().contiguous()
        _step(m, case, be, cfg, t)
        q_static.copy_(li.q[t].cuda())
        if t == 0:
            _step(m, gcase, bg, cfg, 0)           # the first step never reuses: eager
        else:
            if graph is None:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    _step(m, gcase, bg, cfg, 1)
            graph.replay()
        torch.cuda.synchronize()
        for name in ("reuse", "cos", "votes", "ids", "count", "out"):
            a, b = getattr(be, name).cpu().numpy(), getattr(bg, name).cpu().numpy()
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), (t, name)
        reuse = bg.reuse.cpu().numpy()
        qb = W.bf16_bits(gcase.q)
        for b in range(cfg.batch):
            r, c = oracle.selcache(qb[b], q_prev[b], t == 0, cfg.theta)
            if abs(c - cfg.theta) > 1e-9:
                assert bool(reuse[b]) == r, (t, b, c)
        H.check_step(gcase, bg, cfg.k, cfg.n_sink, cfg.n_local, reuse=reuse, prev_ids=prev_ids)
        prev_ids = bg.ids.cpu().numpy().copy()
        all_reused += int(reuse.all())
    assert all_reused > 0, "no step reused every sequence: the skip was never taken"
    status, site = m.ts_get_device_status(bg.ws)
    assert status == m.TS_OK, (status, site)
    del graph
