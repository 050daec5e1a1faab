"""GPU parity of ts_decode_step, the one-call decode step.

ts_decode_step runs the same kernels as ts_selcache -> ts_score -> ts_select ->
ts_sparse_attn except that the vote pass builds the selection's level-1
histogram itself.  Its results must therefore be bit-identical to the four
calls, and (through them) within the oracle contract.  Every case of the
parity suite, three full-size workloads and two selection-cache trajectories
are run both ways."""
import zlib

import numpy as np
import pytest
import torch

import gpu_helpers as H
import oracle
import workloads as W
from test_gpu_parity import CASES, _case

pytestmark = pytest.mark.gpu

NEVER = 2.0   # a cosine threshold that is never reached: every step recomputes


def _fused(case, k, s, l, buf=None, *, theta=NEVER, first_step=True):
    m = H.ts()
    if buf is None:
        buf = m.StepBuffers(case.kv, k, s, l)
    m.ts_decode_step(case.kv, case.q, buf.q_prev, buf.reuse, first_step, theta, k, s, l, buf.votes, buf.ids,
                     buf.count, buf.out, buf.ws, buf.cos)
    torch.cuda.synchronize()
    return buf


def _same(a, b):
    for name in ("votes", "ids", "count", "out", "reuse"):
        x, y = getattr(a, name).cpu().numpy(), getattr(b, name).cpu().numpy()
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), "%s differs between the two paths" % name


@pytest.mark.parametrize("name", sorted(CASES))
def test_case_fused_equals_four_calls(name):
    lengths, h_q, h_kv, d, k, s, l, extra = CASES[name]
    case = _case(lengths, h_q, h_kv, d, seed=zlib.crc32(name.encode()) % 10000, **extra)
    split = H.run_step(case, k, s, l)
    fused = _fused(case, k, s, l)
    _same(split, fused)
    H.check_step(case, fused, k, s, l)


@pytest.mark.parametrize("cfg_name", ["tiny", "qwen7b_32k", "ragged_b32"])
def test_config_fused_full(cfg_name):
    cfg = W.CONFIGS[cfg_name]
    case, _ = H.config_case(cfg)
    fused = _fused(case, cfg.k, cfg.n_sink, cfg.n_local)
    split = H.run_step(case, cfg.k, cfg.n_sink, cfg.n_local)
    _same(split, fused)
    H.check_step(case, fused, cfg.k, cfg.n_sink, cfg.n_local)


def test_repeated_calls_reuse_the_workspace():
    """The selection counters and histogram return to zero after each call: a
    second call on the same workspace gives the same result."""
    cfg = W.CONFIGS["qwen7b_32k"]
    case, _ = H.config_case(cfg)
    buf = _fused(case, cfg.k, cfg.n_sink, cfg.n_local)
    first = {n: getattr(buf, n).clone() for n in ("votes", "ids", "count", "out")}
    for _ in range(3):
        _fused(case, cfg.k, cfg.n_sink, cfg.n_local, buf)
    for n, t in first.items():
        assert torch.equal(getattr(buf, n), t), n


@pytest.mark.parametrize("cfg_name,n", [("llama8b_b4", 4096), ("qwen7b_1m", 16384)])
def test_trajectory_fused_equals_four_calls(cfg_name, n):
    """AR(1) queries with the selection cache on: the fused step and the four
    calls agree bit for bit at every step, and both follow the oracle (its
    reuse decision wherever the cosine is not within 1e-9 of theta)."""
    cfg = W.CONFIGS[cfg_name]
    case, li = H.config_case(cfg, n_override=n)
    m = H.ts()
    bf = m.StepBuffers(case.kv, cfg.k, cfg.n_sink, cfg.n_local)
    bs = m.StepBuffers(case.kv, cfg.k, cfg.n_sink, cfg.n_local)
    q_prev = np.zeros((cfg.batch, cfg.h_q, cfg.head_dim), np.uint16)
    prev_ids = None
    reused = 0
    for t in range(cfg.steps):
        case.q = li.q[t].cuda().contiguous()
        _fused(case, cfg.k, cfg.n_sink, cfg.n_local, bf, theta=cfg.theta, first_step=(t == 0))
        m.ts_selcache(case.q, bs.q_prev, bs.reuse, t == 0, cfg.theta, bs.cos)
        m.ts_score(case.kv, case.q, bs.reuse, bs.votes, bs.ws)
        m.ts_select(case.kv, bs.votes, cfg.k, cfg.n_sink, cfg.n_local, bs.reuse, bs.ids, bs.count, bs.ws)
        m.ts_sparse_attn(case.kv, case.q, bs.ids, bs.count, bs.out, bs.ws)
        torch.cuda.synchronize()
        _same(bs, bf)
        reuse = bf.reuse.cpu().numpy()
        cos = bf.cos.cpu().numpy()
        qb = W.bf16_bits(case.q)
        for b in range(cfg.batch):
            r, c = oracle.selcache(qb[b], q_prev[b], t == 0, cfg.theta)
            assert abs(c - cos[b]) < 1e-12, (t, b, c, cos[b])
            if abs(c - cfg.theta) > 1e-9:
                assert bool(reuse[b]) == r, (t, b, c)
        H.check_step(case, bf, cfg.k, cfg.n_sink, cfg.n_local, reuse=reuse, prev_ids=prev_ids)
        prev_ids = bf.ids.cpu().numpy().copy()
        reused += int(reuse.sum())
    assert reused > 0, "the trajectory never reused a selection"



@pytest.mark.parametrize("cfg_name", ["tiny", "qwen7b_32k", "llama8b_b4", "ragged_b32"])
def test_kernel_count(cfg_name):
    """ts_decode_step_kernels reports the nine kernels of a step (selection
    cache; score pass A, merge, vote pass; collect, resolve, write; attention
    split, merge)."""
    cfg = W.CONFIGS[cfg_name]
    case, _ = H.config_case(cfg, n_override=min(cfg.n, 4096))
    assert H.ts().ts_decode_step_kernels(case.kv, cfg.k, cfg.n_sink, cfg.n_local) == 9
