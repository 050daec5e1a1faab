"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Each pin_* function raises AssertionError when the oracle disagrees with a
hand-worked example (tests/golden/hand_examples.json), a closed form, an
invariant of the definitions, or a brute-force restatement on tiny inputs.
test_oracle_pins.py runs them against the oracle; test_oracle_mutants.py runs
them against deliberately broken copies of the oracle and requires every copy
to fail at least one pin.

Definitions pinned (TokenSelect GitHub README, "Key Takeaways"; GrooveSquid
summary of the TokenSelect paper): per-head Q.K criticality, per-head softmax
over tokens summed over heads (soft vote), top-k selection with sink and local
windows (ties to the lower id), Selection Cache by cosine of consecutive
queries, attention over the selected tokens.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_examples.json")
SCALES = {"ln2/2": math.log(2.0) / 2.0, "ln3/2": math.log(3.0) / 2.0}


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _bits(x) -> np.ndarray:
    """Exact bf16 bits of small integers / floats given as nested lists."""
    t = torch.tensor(x, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float64), torch.tensor(x, dtype=torch.float64)), "not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def _frac(lst):
    return np.array([float(Fraction(s)) for s in lst])


def _rand_case(seed, n, h_q, h_kv, d, dist="normal"):
    k, v = W.random_kv(n, h_kv, d, seed, dist=dist)
    g = torch.Generator().manual_seed(seed + 7)
    q = torch.randn((h_q, d), generator=g).to(torch.bfloat16)
    return W.bf16_bits(k), W.bf16_bits(v), W.bf16_bits(q)


# ---------------------------------------------------------------- scoring


def pin_logits_default_scale():
    c = _golden()["logits_default_scale"]
    k, q = _bits(c["k"]), _bits(c["q"])
    s = oracle.head_logits(k, q, 0)
    assert np.array_equal(s, _frac(c["logits"])), s


def pin_softmax_powers_of_two():
    c = _golden()["softmax_powers_of_two"]
    k, q = _bits(c["k"]), _bits(c["q"])
    s = oracle.head_logits(k, q, 0, SCALES[c["scale"]])
    p, L = oracle.softmax_row(s)
    assert np.allclose(p, _frac(c["p"]), rtol=0, atol=1e-14), p
    assert abs(L - math.log(15.0)) < 1e-13, L          # L = ln(1+2+4+8)


def pin_soft_vote_two_heads():
    c = _golden()["soft_vote_two_heads"]
    v, L = oracle.votes(_bits(c["k"]), _bits(c["q"]), SCALES[c["scale"]])
    assert np.allclose(v, _frac(c["v"]), rtol=0, atol=1e-14), v


def pin_gqa_contiguous_groups():
    c = _golden()["gqa_contiguous_groups"]
    v, L = oracle.votes(_bits(c["k"]), _bits(c["q"]), SCALES[c["scale"]])
    assert np.allclose(v, _frac(c["v"]), rtol=0, atol=1e-14), v


def pin_votes_sum_to_heads():
    """Each head's softmax sums to 1, so the votes sum to h_q."""
    for seed, (n, hq, hk, d) in enumerate([(97, 4, 2, 64), (300, 28, 4, 128), (1, 8, 8, 64),
                                           (513, 6, 3, 64), (64, 32, 8, 128)]):
        k, _, q = _rand_case(seed, n, hq, hk, d)
        v, L = oracle.votes(k, q)
        assert abs(v.sum() - hq) < 1e-12 * hq, (v.sum(), hq)
        assert (v >= 0).all()
        for h in range(hq):
            p, _ = oracle.softmax_row(oracle.head_logits(k, q, h))
            assert abs(p.sum() - 1.0) < 1e-13


def pin_identical_keys_uniform():
    """Identical keys: every head is uniform, v = h_q / n exactly (up to rounding)."""
    k, _ = W.random_kv(50, 2, 64, 3, dist="const")
    q = torch.randn((6, 64), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    v, _ = oracle.votes(W.bf16_bits(k), W.bf16_bits(q))
    assert np.allclose(v, 6.0 / 50.0, rtol=1e-14, atol=0), v


def pin_single_token():
    k, _, q = _rand_case(11, 1, 4, 2, 64)
    v, _ = oracle.votes(k, q)
    assert v.shape == (1,) and abs(v[0] - 4.0) < 1e-14


def pin_large_logits_stable():
    """Logits in the thousands: the max shift keeps the softmax finite."""
    k = _bits([[[60.0] * 64], [[59.0] * 64], [[-60.0] * 64]])
    q = _bits([[60.0] * 64])
    v, L = oracle.votes(k, q)
    assert np.isfinite(v).all() and abs(v.sum() - 1.0) < 1e-12
    # logits are 60*60*64/8 = 28800, 28320 and -28800: the last is e^-57600 below -> 0
    assert abs(v[0] - 1.0) < 1e-12 and v[2] == 0.0
    assert abs(L[0] - 28800.0) < 1e-9


def pin_strided_layout():
    """A padded layout (junk 1e4 in the gaps) gives the same results as the dense one."""
    n, hk, d, hq = 77, 2, 64, 4
    kd, vd = W.random_kv(n, hk, d, 21)
    kp, vp = W.random_kv(n, hk, d, 21, stride_tok=3 * hk * d + 8, stride_head=d + 40)
    assert torch.equal(kd.float(), kp.float()) and torch.equal(vd.float(), vp.float())
    q = torch.randn((hq, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    qb = W.bf16_bits(q)
    a, La = oracle.votes(W.bf16_bits(kd), qb)
    b, Lb = oracle.votes(W.bf16_bits(kp), qb)
    assert np.array_equal(a, b) and np.array_equal(La, Lb)
    ids = np.array([0, 5, 9, 40, 76], np.int32)
    oa = oracle.sparse_attn(W.bf16_bits(kd), W.bf16_bits(vd), qb, ids)
    ob = oracle.sparse_attn(W.bf16_bits(kp), W.bf16_bits(vp), qb, ids)
    assert np.array_equal(oa, ob)


# ---------------------------------------------------------------- selection


def _brute_select(v, k, s, l):
    """Rank counting: candidate i is in T iff fewer than k candidates precede it
    in (vote desc, id asc) order.  O(n^2), no sorting."""
    n = v.size
    s_end = min(s, n)
    l0 = max(n - l, s_end)
    chosen = np.zeros(n, bool)
    chosen[:s_end] = True
    chosen[l0:] = True
    c = np.arange(s_end, l0)
    if c.size and k > 0:
        vc = v[c]
        before = (vc[None, :] > vc[:, None]) | ((vc[None, :] == vc[:, None]) & (c[None, :] < c[:, None]))
        rank = before.sum(axis=1)
        chosen[c[rank < k]] = True
    return np.nonzero(chosen)[0].astype(np.int32)


def pin_select_hand_example():
    c = _golden()["select_with_ties"]
    ids, m = oracle.select(np.array(c["votes"], np.float64), c["k"], c["n_sink"], c["n_local"])
    assert m == c["count"] and ids.tolist() == c["ids"], (ids, m)


def pin_windows():
    for n, s, l, se, lb in _golden()["windows"]["cases"]:
        assert oracle.windows(n, s, l) == (se, lb), (n, s, l, oracle.windows(n, s, l))


def pin_select_brute_force(seeds=1000):
    rng = np.random.default_rng(12345)
    for _ in range(seeds):
        n = int(rng.integers(0, 65))
        k = int(rng.integers(0, 24))
        s = int(rng.integers(0, 6))
        l = int(rng.integers(0, 10))
        v = np.round(rng.random(n) * rng.choice([4, 16, 1 << 20])) / 8.0   # many ties
        ids, m = oracle.select(v, k, s, l)
        want = _brute_select(v, k, s, l)
        assert m == want.size and np.array_equal(ids[:m], want), (n, k, s, l)
        assert (ids[m:] == -1).all()


def pin_select_all_equal():
    """All-equal votes: the tie-break takes the lowest candidate ids."""
    n, k, s, l = 40, 7, 3, 5
    ids, m = oracle.select(np.full(n, 0.25), k, s, l)
    want = list(range(0, s)) + list(range(s, s + k)) + list(range(n - l, n))
    assert m == len(want) and ids[:m].tolist() == want


def pin_select_counts():
    for n, k, s, l in [(100, 10, 4, 20), (20, 10, 4, 20), (24, 10, 4, 20), (30, 10, 4, 20),
                       (0, 5, 1, 1), (5, 0, 0, 0), (50, 100, 0, 0)]:
        ids, m = oracle.select(np.linspace(0, 1, n), k, s, l)
        assert m == min(n, k + s + l), (n, k, s, l, m)
        assert np.all(np.diff(ids[:m]) > 0)


def pin_planted_keys_selected():
    """Planted query-aligned keys carry the top votes and are always selected."""
    cfg = W.CONFIGS["tiny"]
    li = W.layer_inputs(cfg)
    k, q = W.bf16_bits(li.k), W.bf16_bits(li.q[0, 0])
    v, _ = oracle.votes(k, q)
    ids, m = oracle.select(v, cfg.k, cfg.n_sink, cfg.n_local)
    assert set(li.planted[0].tolist()) <= set(ids[:m].tolist())
    top = np.argsort(-v, kind="stable")[:len(li.planted[0])]
    assert set(top.tolist()) == set(li.planted[0].tolist())


# ---------------------------------------------------------------- attention


def pin_attention_two_tokens():
    c = _golden()["attention_two_tokens"]
    out = oracle.sparse_attn(_bits(c["k"]), _bits(c["v"]), _bits(c["q"]),
                             np.array([0, 1], np.int32), scale=SCALES[c["scale"]])
    want = np.array([[float(Fraction(x)) for x in row] for row in c["out"]])
    assert np.allclose(out, want, rtol=0, atol=1e-13), out
    dense = oracle.dense_attn(_bits(c["k"]), _bits(c["v"]), _bits(c["q"]), scale=SCALES[c["scale"]])
    assert np.allclose(dense, want, rtol=0, atol=1e-13), dense


def pin_attention_single_row():
    """One selected row: every head's output is that row of its kv head's V."""
    k, v, q = _rand_case(31, 20, 6, 3, 64)
    for j in (0, 7, 19):
        out = oracle.sparse_attn(k, v, q, np.array([j], np.int32))
        vf = torch.from_numpy(v.astype(np.int16)).view(torch.bfloat16).double().numpy()
        for h in range(6):
            assert np.array_equal(out[h], vf[j, h // 2]), (j, h)


def pin_full_selection_is_dense():
    """k >= |candidates| selects every token: sparse attention = dense attention."""
    for seed, (n, hq, hk, d) in enumerate([(90, 4, 2, 64), (33, 28, 4, 128), (5, 2, 2, 64)]):
        k, v, q = _rand_case(40 + seed, n, hq, hk, d)
        vv, _ = oracle.votes(k, q)
        ids, m = oracle.select(vv, n, 4, 8)
        assert m == n
        sp = oracle.sparse_attn(k, v, q, ids, m)
        de = oracle.dense_attn(k, v, q)
        assert np.allclose(sp, de, rtol=0, atol=1e-12)


def pin_mha_is_per_head():
    """h_q == h_kv: each head attends with its own K/V head only."""
    k, v, q = _rand_case(51, 30, 3, 3, 64)
    ids = np.arange(0, 30, 3, dtype=np.int32)
    full = oracle.sparse_attn(k, v, q, ids)
    for h in range(3):
        one = oracle.sparse_attn(np.ascontiguousarray(k[:, h:h + 1]), np.ascontiguousarray(v[:, h:h + 1]),
                                 np.ascontiguousarray(q[h:h + 1]), ids)
        assert np.array_equal(full[h], one[0])


# ---------------------------------------------------------------- selection cache


def pin_selcache_cases():
    a = _bits([1.0, 0.0, 0.0, 0.0])
    b = _bits([1.0, 1.0, 0.0, 0.0])
    o = _bits([0.0, 1.0, 0.0, 0.0])
    assert abs(oracle.cosine(a, b) - 1.0 / math.sqrt(2.0)) < 1e-15
    assert oracle.cosine(a, o) == 0.0
    q = W.bf16_bits(torch.randn(3, 64, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16))
    neg = (q ^ np.uint16(0x8000))                      # bf16 sign flip: -q exactly
    assert abs(oracle.cosine(q, q) - 1.0) < 1e-15
    assert abs(oracle.cosine(q, neg) + 1.0) < 1e-15

    prev = q.copy().reshape(-1)
    r, c = oracle.selcache(q, prev, first_step=False, theta=0.9)
    assert r and abs(c - 1.0) < 1e-15
    prev = neg.copy().reshape(-1)
    r, c = oracle.selcache(q, prev, first_step=False, theta=0.9)
    assert (not r) and abs(c + 1.0) < 1e-15
    assert np.array_equal(prev, q.reshape(-1)), "q_prev must hold the current query afterwards"
    prev = q.copy().reshape(-1)
    r, c = oracle.selcache(q, prev, first_step=True, theta=-2.0)
    assert not r, "the first step never reuses"
    # "at or above": cosine exactly equal to theta reuses
    prev = o.copy()
    r, c = oracle.selcache(a, prev, first_step=False, theta=0.0)
    assert r and c == 0.0
    prev = o.copy()
    r, c = oracle.selcache(a, prev, first_step=False, theta=1e-9)
    assert not r


def pin_ar1_reuse_rate():
    """AR(1) queries q_t = rho q_{t-1} + e_t: the flattened cosine of consecutive
    queries tends to rho*sqrt(V_{t-1}/V_t) with V_t = sum_{j<=t} rho^(2j)."""
    cfg = W.CONFIGS["llama8b_b4"]
    qs = W.queries(cfg)
    T = qs.shape[0]
    rho = cfg.ar_rho
    prev = W.bf16_bits(qs[0]).copy()
    got = np.zeros((T, cfg.batch))
    for t in range(1, T):
        cur = W.bf16_bits(qs[t])
        for b in range(cfg.batch):
            _, got[t, b] = oracle.selcache(cur[b], prev[b], False, cfg.theta)
    Vt = np.cumsum(rho ** (2 * np.arange(T)))
    want = rho * np.sqrt(Vt[:-1] / Vt[1:])
    err = np.abs(got[1:].mean(axis=1) - want)
    assert err.max() < 0.04, err.max()            # per-decision noise ~ 1/sqrt(h_q d) = 0.016
    reuse = (got[1:] >= cfg.theta).mean()
    assert 0.80 < reuse < 0.95, reuse



# ------------------------------------------------ decode loop with KV append (R19)

def _rand_query(seed, h_q, d):
    g = torch.Generator().manual_seed(seed)
    return W.bf16_bits(torch.randn((h_q, d), generator=g).to(torch.bfloat16))


def pin_reuse_hand_example():
    """The hand-worked growth, shrink and unchanged-length cases."""
    c = _golden()["reuse_with_growth"]
    v = np.array(c["votes"], np.float64)
    ids, m = oracle.select(v, c["k"], c["n_sink"], c["n_local"])
    assert m == c["step0"]["count"] and ids[:m].tolist() == c["step0"]["ids"], (ids, m)
    for r in c["reused"]:
        got, gm = oracle.reuse_ids(ids, m, r["n_old"], r["n_new"], c["k"], c["n_sink"], c["n_local"])
        assert gm == r["count"] and got[:gm].tolist() == r["ids"] and (got[gm:] == -1).all(), (r, got, gm)
    t = c["tiny_then_grow"]
    got, gm = oracle.reuse_ids(np.array(t["prev_ids"], np.int32), t["prev_count"], t["n_old"], t["n_new"], c["k"],
                               c["n_sink"], c["n_local"])
    assert gm == t["count"] and got[:gm].tolist() == t["ids"], (got, gm)


def pin_reuse_unchanged_length_keeps_row():
    """With the same length the reused row is exactly the previous row (R8)."""
    rng = np.random.default_rng(777)
    for _ in range(300):
        n = int(rng.integers(0, 80))
        k, s, l = int(rng.integers(0, 20)), int(rng.integers(0, 6)), int(rng.integers(0, 12))
        ids, m = oracle.select(np.round(rng.random(n) * 8) / 8, k, s, l)
        got, gm = oracle.reuse_ids(ids, m, n, n, k, s, l)
        assert gm == m and np.array_equal(got, ids), (n, k, s, l)


def pin_reuse_growth_properties():
    """After growth from n0 to n1 >= n0: the windows of n1 are in the row, every
    other id was selected at n0 (it is from the old top-k part, which rank
    counting finds independently), the old top-k part is kept whole, and
    growing in two steps gives the same row as growing in one."""
    rng = np.random.default_rng(4242)
    for _ in range(400):
        n0 = int(rng.integers(0, 70))
        n1 = n0 + int(rng.integers(0, 12))
        n2 = n1 + int(rng.integers(0, 12))
        k, s, l = int(rng.integers(0, 20)), int(rng.integers(0, 6)), int(rng.integers(0, 12))
        v = np.round(rng.random(n0) * 8) / 8
        ids, m = oracle.select(v, k, s, l)
        got, gm = oracle.reuse_ids(ids, m, n0, n1, k, s, l)
        row = got[:gm]
        assert (got[gm:] == -1).all() and np.all(np.diff(row) > 0) and (gm == 0 or row[-1] < n1)
        s1, l1 = min(s, n1), max(n1 - l, min(s, n1))
        assert set(range(s1)) <= set(row.tolist()) and set(range(l1, n1)) <= set(row.tolist())
        s0, l0 = min(s, n0), max(n0 - l, min(s, n0))
        top_old = {int(i) for i in _brute_select(v, k, s, l) if s0 <= i < l0}
        middle = {int(i) for i in row if s1 <= i < l1}
        assert middle == top_old, (n0, n1, k, s, l)          # growth never pushes a kept id out
        two, tm = oracle.reuse_ids(got, gm, n1, n2, k, s, l)
        one, om = oracle.reuse_ids(ids, m, n0, n2, k, s, l)
        assert tm == om and np.array_equal(two, one), (n0, n1, n2, k, s, l)


def pin_decode_loop_slides_the_local_window():
    """A decode loop that reuses at every step after the first keeps the first
    step's top-k part, and its local window follows the growing cache: the
    last n_local ids of step t are n_t - n_local .. n_t - 1."""
    d, h_q, h_kv, n0, T = 16, 4, 2, 200, 6
    k, v, _ = _rand_case(31, n0 + T, h_q, h_kv, d)
    qs = np.stack([_rand_query(90 + t, h_q, d) for t in range(T)])
    kt, s, l = 12, 3, 8
    steps = oracle.decode_loop(k, v, n0, qs, kt, s, l, theta=0.9, reuse_override=[False] + [True] * (T - 1))
    first = steps[0]
    top0 = [int(i) for i in first["ids"][:first["count"]] if s <= i < n0 - l]
    assert len(top0) == kt
    for t, st in enumerate(steps):
        row = st["ids"][:st["count"]].tolist()
        assert st["n"] == n0 + t and st["count"] == kt + s + l
        assert row[:s] == list(range(s)) and row[s:s + kt] == top0 and row[-l:] == list(range(n0 + t - l, n0 + t))


def pin_decode_loop_without_reuse_is_a_fresh_step():
    """Without reuse every step is the single-step oracle over the current
    prefix of the cache: the loop appends before it attends."""
    d, h_q, h_kv, n0, T = 16, 4, 2, 120, 4
    k, v, _ = _rand_case(77, n0 + T, h_q, h_kv, d)
    qs = np.stack([_rand_query(500 + t, h_q, d) for t in range(T)])
    steps = oracle.decode_loop(k, v, n0, qs, 10, 2, 6, theta=2.0)
    for t, st in enumerate(steps):
        n = n0 + t
        assert not st["reuse"]
        ref = oracle.decode_step(k[:n], v[:n], np.array([0, n]), qs[t][None], 10, 2, 6)
        assert st["count"] == ref.count[0] and np.array_equal(st["ids"], ref.ids[0])
        assert np.array_equal(st["out"], ref.out[0])


# ------------------------------------------- page-level comparator (Quest)
# Bohrium page for Quest (arXiv 2406.10774), Abstract and "Method Overview"
# (4): per-page min/max keys, a query-dependent upper-bound criticality per
# page, the Top-K pages loaded for attention.


def pin_quest_hand_example():
    c = _golden()["quest_pages"]
    kb = _bits(c["keys"]).reshape(len(c["keys"]), 1, 4)
    qb = _bits(c["q"])
    kmin, kmax = oracle.quest_meta(kb, c["page_size"])
    assert np.array_equal(kmin.reshape(-1, 4), _bits(c["kmin"])), kmin
    assert np.array_equal(kmax.reshape(-1, 4), _bits(c["kmax"])), kmax
    sc = oracle.quest_scores(kmin, kmax, qb)
    assert np.array_equal(sc, _frac(c["scores"])), sc
    for case in c["select"]:
        ids, m = oracle.quest_select(sc, len(c["keys"]), c["page_size"], case["k"], c["n_sink"], c["n_local"])
        assert m == case["count"] and ids[:m].tolist() == case["ids"], (ids, m)


def _pages_np(kf, P):
    """[pages] list of float64 [tokens, h_kv, d] slices (numpy slicing only)."""
    n = kf.shape[0]
    return [kf[j * P:min((j + 1) * P, n)] for j in range(-(-n // P))]


def pin_quest_meta_is_the_page_box():
    """Every key of a page lies in [kmin, kmax] and each bound is the value of
    some key of that page (the extremes over exactly the page's tokens, the
    short last page included); against numpy's min / max of the slices."""
    for seed, n, h_kv, d, P in [(1, 100, 2, 64, 16), (2, 33, 4, 128, 8), (3, 7, 1, 64, 4), (4, 64, 2, 64, 64),
                                (5, 5, 2, 64, 128)]:
        kb, _, _ = _rand_case(seed, n, 2 * h_kv, h_kv, d)
        kmin, kmax = oracle.quest_meta(kb, P)
        kf = kb.astype(np.uint32) << 16
        kf = kf.view(np.float32).astype(np.float64)
        pages = _pages_np(kf, P)
        assert kmin.shape == (len(pages), h_kv, d)
        for j, pg in enumerate(pages):
            lo = (kmin[j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            hi = (kmax[j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            assert np.array_equal(lo, pg.min(axis=0)), (seed, j)
            assert np.array_equal(hi, pg.max(axis=0)), (seed, j)


def pin_quest_one_token_pages_are_summed_logits():
    """Pages of one token: the box is the key itself, so the page score is the
    exact sum over query heads of the scaled dot products with that key."""
    for seed, n, h_q, h_kv, d in [(11, 50, 8, 2, 64), (12, 20, 28, 4, 128), (13, 9, 4, 4, 64)]:
        kb, _, qb = _rand_case(seed, n, h_q, h_kv, d)
        kmin, kmax = oracle.quest_meta(kb, 1)
        sc = oracle.quest_scores(kmin, kmax, qb)
        kf = (kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qf = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        G = h_q // h_kv
        want = np.zeros(n)
        for h in range(h_q):
            want += (kf[:, h // G, :] @ qf[h]) / math.sqrt(d)
        assert np.allclose(sc, want, rtol=1e-12, atol=1e-12), (seed, np.abs(sc - want).max())


def pin_quest_score_bounds_every_key():
    """The page score bounds the head-summed scaled logit of every key of the
    page, and is reached when the page's keys include the corner of the box
    that each query head prefers (a page of one key per channel sign pattern
    is not needed: a page of identical keys reaches it)."""
    for seed, n, h_q, h_kv, d, P in [(21, 200, 8, 2, 64, 16), (22, 97, 28, 4, 128, 32), (23, 40, 4, 1, 64, 8)]:
        kb, _, qb = _rand_case(seed, n, h_q, h_kv, d)
        kmin, kmax = oracle.quest_meta(kb, P)
        sc = oracle.quest_scores(kmin, kmax, qb)
        kf = (kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qf = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        G = h_q // h_kv
        summed = np.zeros(n)
        for h in range(h_q):
            summed += (kf[:, h // G, :] @ qf[h]) / math.sqrt(d)
        for j in range(sc.size):
            tok = summed[j * P:(j + 1) * P]
            assert (tok <= sc[j] + 1e-9 * (1 + abs(sc[j]))).all(), (seed, j)
        # identical keys in a page: the box is a point and the bound is exact
        kb2 = np.repeat(kb[::P], P, axis=0)[:n]
        sc2 = oracle.quest_scores(*oracle.quest_meta(kb2, P), qb)
        kf2 = (kb2.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        s2 = np.zeros(n)
        for h in range(h_q):
            s2 += (kf2[:, h // G, :] @ qf[h]) / math.sqrt(d)
        assert np.allclose(sc2, s2[::P], rtol=1e-12, atol=1e-12), seed


def _brute_quest_select(sc, n, P, k, s, l):
    """Rank counting over candidate pages: page j is chosen iff fewer than
    floor(k / P) candidate pages precede it in (score desc, page asc) order."""
    s_end = min(s, n)
    l0 = max(n - l, s_end)
    chosen = np.zeros(n, bool)
    chosen[:s_end] = True
    chosen[l0:] = True
    pages = np.arange(-(-n // P)) if n > 0 else np.arange(0)
    cand = np.array([j for j in pages if max(j * P, s_end) < min((j + 1) * P, l0)], np.int64)
    kp = k // P
    if cand.size and kp > 0:
        v = sc[cand]
        before = (v[None, :] > v[:, None]) | ((v[None, :] == v[:, None]) & (cand[None, :] < cand[:, None]))
        for j in cand[before.sum(axis=1) < kp]:
            chosen[max(j * P, s_end):min((j + 1) * P, l0)] = True
    return np.nonzero(chosen)[0].astype(np.int32)


def pin_quest_select_brute_force(seeds=600):
    rng = np.random.default_rng(2406)
    for _ in range(seeds):
        n = int(rng.integers(0, 90))
        P = int(rng.choice([1, 2, 4, 8, 16]))
        k = int(rng.integers(0, 40))
        s = int(rng.integers(0, 9))
        l = int(rng.integers(0, 20))
        sc = np.round(rng.standard_normal(-(-n // P)) * rng.choice([2, 8, 1 << 20])) / 4.0   # ties
        ids, m = oracle.quest_select(sc, n, P, k, s, l)
        want = _brute_quest_select(sc, n, P, k, s, l)
        assert m == want.size and np.array_equal(ids[:m], want), (n, P, k, s, l)
        assert (ids[m:] == -1).all() and m <= min(n, k + s + l)


def pin_quest_one_token_pages_select_like_tokens():
    """With one-token pages the page selection is the token-level top-k of the
    same scores."""
    rng = np.random.default_rng(7)
    for n, k, s, l in [(300, 40, 4, 32), (50, 100, 2, 2), (64, 0, 4, 8)]:
        sc = rng.standard_normal(n)
        a = oracle.quest_select(sc, n, 1, k, s, l)
        b = oracle.select(sc, k, s, l)
        assert a[1] == b[1] and np.array_equal(a[0], b[0])


def pin_quest_planted_pages_selected():
    """Keys planted along the query dominate their pages' bounds: the pages
    holding them are chosen."""
    cfg = W.CONFIGS["tiny"]
    li = W.layer_inputs(cfg)
    kb, qb = W.bf16_bits(li.k), W.bf16_bits(li.q[0, 0])
    P = 16
    sc = oracle.quest_scores(*oracle.quest_meta(kb, P), qb)
    ids, m = oracle.quest_select(sc, kb.shape[0], P, cfg.k, cfg.n_sink, cfg.n_local)
    assert set(li.planted[0].tolist()) <= set(ids[:m].tolist())


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
