"""Decode loop with KV append on a growing cache (one sequence, capacity
mode): before each step one token is appended on the device (ts_append_kv),
then one ts_decode_step runs with the selection cache on.  Checked against
the oracle's decode loop (reading R19: a reused selection keeps its top-k part
and takes the sink and local windows of the grown cache), eagerly and as a
replayed CUDA graph of [append, step] (bit-identical to the eager loop)."""
import dataclasses

import numpy as np
import pytest
import torch

import gpu_helpers as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu

N0, T = 3000, 14
K_TOP, SINK, LOCAL = 256, 4, 64
THETA = 0.9


def _inputs():
    cfg = dataclasses.replace(W.CONFIGS["qwen7b_32k"], n=N0 + T, steps=T, ar_rho=0.95, theta=THETA)
    k, v = W.random_kv(N0 + T, cfg.h_kv, cfg.head_dim, 4321, device="cuda")
    qs = W.queries(cfg)                      # [T, 1, h_q, d] bf16, AR(1)
    return cfg, k, v, qs


def _loop(cfg, k, v, qs, graph: bool):
    m = H.ts()
    kbuf, vbuf = torch.zeros_like(k), torch.zeros_like(v)
    kbuf[:N0], vbuf[:N0] = k[:N0], v[:N0]
    kv = m.KVCache(kbuf, vbuf, np.array([0, N0]), cfg.h_q, capacity=N0 + T)
    buf = m.StepBuffers(kv, K_TOP, SINK, LOCAL)
    q = qs[0].cuda().contiguous()
    k_new = torch.empty_like(k[0])
    v_new = torch.empty_like(v[0])
    recs = []

    def step(first):
        m.ts_decode_step(kv, q, buf.q_prev, buf.reuse, first, THETA, K_TOP, SINK, LOCAL, buf.votes, buf.ids,
                         buf.count, buf.out, buf.ws, buf.cos)

    def append_and_step():
        m.ts_append_kv(kv, k_new, v_new, buf.ws)
        step(False)

    g = None
    for t in range(T):
        q.copy_(qs[t].cuda())
        if t == 0:
            step(True)
        else:
            k_new.copy_(k[N0 + t - 1])
            v_new.copy_(v[N0 + t - 1])
            if graph:
                if g is None:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        append_and_step()
                g.replay()
            else:
                append_and_step()
        torch.cuda.synchronize()
        recs.append({"n": int(kv.seq_offsets_dev[1].item()), "reuse": bool(buf.reuse.item()),
                     "cos": float(buf.cos.item()), "votes": buf.votes.cpu().numpy().copy(),
                     "ids": buf.ids.cpu().numpy()[0].copy(), "count": int(buf.count.item()),
                     "out": buf.out.cpu().numpy()[0].copy()})
    status, site = m.ts_get_device_status(buf.ws)
    assert status == m.TS_OK, (status, site)
    return recs


@pytest.fixture(scope="module")
def loops():
    cfg, k, v, qs = _inputs()
    return cfg, k, v, qs, _loop(cfg, k, v, qs, graph=False), _loop(cfg, k, v, qs, graph=True)


def test_eager_loop_follows_the_oracle(loops):
    cfg, k, v, qs, eager, _ = loops
    kb, vb, qb = W.bf16_bits(k), W.bf16_bits(v), W.bf16_bits(qs)
    reuse = [r["reuse"] for r in eager]
    ref = oracle.decode_loop(kb, vb, N0, qb[:, 0], K_TOP, SINK, LOCAL, THETA, reuse_override=reuse)
    prev = None
    for t, (g, o) in enumerate(zip(eager, ref)):
        assert g["n"] == N0 + t
        if abs(o["cos"] - THETA) > 1e-9:
            assert g["reuse"] == (o["cos"] >= THETA and t > 0), (t, o["cos"])
        if t > 0:
            assert abs(g["cos"] - o["cos"]) < 1e-12, (t, g["cos"], o["cos"])
        n = g["n"]
        if g["reuse"]:
            # the rule applied to the GPU's own previous row
            want, wm = oracle.reuse_ids(prev["ids"], prev["count"], prev["n"], n, K_TOP, SINK, LOCAL)
            assert g["count"] == wm and np.array_equal(g["ids"], want), t
        else:
            H.check_votes(g["votes"][:n], o["votes"], cfg.h_q)
            H.check_ids(g["ids"], g["count"], o["ids"], o["count"], o["votes"], n, K_TOP, SINK, LOCAL)
        o_ref = oracle.sparse_attn(kb[:n], vb[:n], qb[t, 0], g["ids"], g["count"])
        assert np.abs(g["out"] - o_ref).max() <= H.OUT_ATOL, t
        prev = g
    assert any(reuse), "the loop never reused a selection"
    assert not all(reuse[1:]), "the loop never recomputed a selection after the first step"


def test_graph_loop_equals_eager(loops):
    _, _, _, _, eager, graph = loops
    for t, (a, b) in enumerate(zip(eager, graph)):
        for key in ("n", "reuse", "count"):
            assert a[key] == b[key], (t, key)
        for key in ("ids", "out", "votes"):
            assert np.array_equal(a[key].view(np.uint8), b[key].view(np.uint8)), (t, key)


def test_append_to_a_full_cache_is_reported():
    m = H.ts()
    k, v = W.random_kv(8, 4, 128, 5, device="cuda")
    kv = m.KVCache(k, v, np.array([0, 8]), 28, capacity=8)
    buf = m.StepBuffers(kv, 4, 1, 1)
    m.ts_append_kv(kv, k[0].contiguous(), v[0].contiguous(), buf.ws)
    torch.cuda.synchronize()
    assert int(kv.seq_offsets_dev[1].item()) == 8
    status, _ = m.ts_get_device_status(buf.ws)
    assert status == m.TS_ERR_INVALID_ARG
