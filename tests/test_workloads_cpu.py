"""The synthetic inputs follow the workload recipe: shapes and selection sizes,
ragged lengths, AR(1) queries, lognormal key-channel scales and planted
query-aligned keys (checked statistically on the generated data)."""
import math

import numpy as np
import torch

import workloads as W


def test_configs_match_the_recipe():
    c = W.CONFIGS
    assert (c["tiny"].batch, c["tiny"].h_q, c["tiny"].h_kv, c["tiny"].head_dim, c["tiny"].n) == (1, 4, 2, 64, 4096)
    assert (c["tiny"].k, c["tiny"].n_sink, c["tiny"].n_local, c["tiny"].planted_count) == (256, 4, 64, 16)
    q = c["qwen7b_32k"]
    assert (q.batch, q.h_q, q.h_kv, q.head_dim, q.n, q.k, q.n_sink, q.n_local) == (1, 28, 4, 128, 32768, 2048, 4, 512)
    assert q.k_lognormal_sigma == 0.5 and q.planted_frac == 0.01 and q.theta is None
    l = c["llama8b_b4"]
    assert (l.batch, l.h_q, l.h_kv, l.head_dim, l.n, l.k, l.n_sink, l.n_local) == (4, 32, 8, 128, 131072, 2048, 4, 512)
    assert (l.steps, l.theta, l.ar_rho, l.planted_frac, l.planted_count) == (64, 0.9, 0.95, 0.0, 0)
    r = c["ragged_b32"]
    assert (r.batch, r.h_q, r.h_kv, r.head_dim, r.n_min, r.n, r.k, r.n_sink, r.n_local) == \
        (32, 32, 8, 128, 8192, 65536, 1024, 4, 256)
    assert r.planted_frac == 0.005
    m = c["qwen7b_1m"]
    assert (m.batch, m.h_q, m.h_kv, m.head_dim, m.n, m.layers, m.k, m.n_sink, m.n_local) == \
        (1, 28, 4, 128, 1048576, 28, 4096, 4, 1024)
    assert (m.steps, m.theta, m.ar_rho, m.k_lognormal_sigma, m.planted_frac) == (16, 0.9, 0.95, 0.5, 0.001)
    assert W._planted_count(q, q.n) == 327 and W._planted_count(m, m.n) == 1048


def test_ragged_lengths_are_uniform_in_range_and_seeded():
    a = W.seq_lengths(W.CONFIGS["ragged_b32"])
    assert a.size == 32 and a.min() >= 8192 and a.max() <= 65536
    assert np.array_equal(a, W.seq_lengths(W.CONFIGS["ragged_b32"]))
    off = W.seq_offsets(a)
    assert off[0] == 0 and np.array_equal(np.diff(off), a)


def test_ar1_queries_have_unit_innovations():
    cfg = W.CONFIGS["llama8b_b4"]
    q = W.queries(cfg).to(torch.float64).numpy()          # [64, 4, 32, 128], rounded to bf16
    e = q[1:] - cfg.ar_rho * q[:-1]                        # innovations (+ bf16 rounding)
    assert abs(e.mean()) < 0.01 and abs(e.std() - 1.0) < 0.02, (e.mean(), e.std())
    assert abs(q[0].std() - 1.0) < 0.03
    # the stationary variance 1 / (1 - rho^2) is approached along the chain
    assert abs(q[-1].var() - (1 - cfg.ar_rho ** 128) / (1 - cfg.ar_rho ** 2)) < 1.0


def test_lognormal_channel_scales_and_planted_keys():
    cfg = W.CONFIGS["qwen7b_32k"]
    li = W.layer_inputs(cfg, 0, "cpu")
    k = li.k.to(torch.float64)
    pos = li.planted[0]
    assert pos.size == 327 and np.unique(pos).size == 327 and pos.min() >= 0 and pos.max() < cfg.n
    mask = np.ones(cfg.n, bool)
    mask[pos] = False
    kk = k[torch.from_numpy(mask)]                         # unplanted rows: N(0, 1) * scale[g, c]
    log_std = torch.log(kk.std(dim=0)).numpy().ravel()     # one value per (kv head, channel)
    assert abs(log_std.mean()) < 0.1 and abs(log_std.std() - 0.5) < 0.06, (log_std.mean(), log_std.std())
    # planted rows: 3 sqrt(d) qbar_g / |qbar_g| + N(0, 0.1): norm ~ 3 sqrt(d), aligned with qbar_g
    q0 = li.q[0, 0].to(torch.float64).reshape(cfg.h_kv, cfg.group, cfg.head_dim).mean(dim=1)
    kp = k[torch.from_numpy(pos)]                          # [327, h_kv, d]
    norms = kp.norm(dim=2)
    assert torch.allclose(norms, torch.full_like(norms, 3 * math.sqrt(cfg.head_dim)), rtol=0.02)
    cos = (kp * q0.unsqueeze(0)).sum(dim=2) / (norms * q0.norm(dim=1).unsqueeze(0))
    assert cos.min() > 0.99
