"""Token-axis split of one sequence (query_aware_kv_ts_b200.split), its
kernels on one GPU: the sequence is cut into shards, the phases run per shard
in one process with the all-gathers done as copies, and the joined result is
compared with the oracle's single-sequence step and with the one-GPU
ts_decode_step of the whole sequence.

Checks: each shard's votes against the oracle's votes of the whole sequence
(1e-3 relative); the union of the shards' selections (as sequence ids)
exactly equal to the oracle's selection taken on the GPU's own fp32 votes, and
to the oracle's float64 selection outside the 1e-6 band; the joined attention
output within 2e-3 of the oracle's attention over that union."""
import numpy as np
import pytest
import torch

import gpu_helpers as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    # name: (n, h_q, h_kv, d, k, sink, local, shard lengths)
    "qwen_shape_two_shards": (5000, 28, 4, 128, 512, 4, 128, [2500, 2500]),
    "qwen_shape_uneven_four": (6000, 28, 4, 128, 512, 4, 128, [1, 1999, 3000, 1000]),
    "llama_shape_three": (4096, 32, 8, 128, 256, 4, 64, [1000, 2048, 1048]),
    "tiny_shard_in_sink": (3000, 4, 2, 64, 128, 16, 32, [3, 10, 2987]),
    "shard_in_local_window": (3000, 8, 2, 128, 100, 4, 300, [2800, 150, 50]),
    "budget_above_candidates": (600, 8, 2, 64, 1000, 4, 16, [300, 300]),
    "one_shard": (2000, 28, 4, 128, 256, 4, 64, [2000]),
}


def _run(name):
    n, h_q, h_kv, d, k, s, l, lens = CASES[name]
    assert sum(lens) == n
    kk, vv = W.random_kv(n, h_kv, d, 7 + n, device="cuda")
    q = torch.randn((1, h_q, d), generator=torch.Generator().manual_seed(n)).to(torch.bfloat16).cuda()
    m = H.ts()
    from query_aware_kv_ts_b200 import split
    shards, t = [], 0
    for ln in lens:
        kv = m.KVCache(kk[t:t + ln], vv[t:t + ln], np.array([0, ln]), h_q)
        shards.append((kv, split.ShardBuffers(kv, k, s, l, len(lens)), t))
        t += ln
    out = split.emulate_split_decode_step(shards, q, n)
    torch.cuda.synchronize()
    return (n, h_q, h_kv, d, k, s, l, lens), kk, vv, q, shards, out


@pytest.mark.parametrize("name", sorted(CASES))
def test_split_matches_oracle(name):
    (n, h_q, h_kv, d, k, s, l, lens), kk, vv, q, shards, out = _run(name)
    kb, vb, qb = W.bf16_bits(kk), W.bf16_bits(vv), W.bf16_bits(q)[0]
    v_ref, _ = oracle.votes(kb, qb)
    votes = np.concatenate([b.step.votes.cpu().numpy()[:kv.n_total] for kv, b, _ in shards])
    H.check_votes(votes, v_ref, h_q)
    # the union of the shards' rows, as sequence ids
    union = []
    for kv, b, t in shards:
        c = int(b.step.count.cpu().numpy()[0])
        union += [int(x) + t for x in b.step.ids.cpu().numpy()[0][:c]]
    union = np.array(sorted(union), np.int32)
    assert np.all(np.diff(union) > 0)
    want, m_ = oracle.select(votes.astype(np.float64), k, s, l)
    assert union.size == m_ and np.array_equal(union, want[:m_]), "selection differs on the GPU's own votes"
    ref_ids, ref_m = oracle.select(v_ref, k, s, l)
    H.check_ids(np.concatenate([union, -np.ones(k + s + l - union.size, np.int32)]), union.size, ref_ids, ref_m,
                v_ref, n, k, s, l)
    o_ref = oracle.sparse_attn(kb, vb, qb, union, union.size)
    err = float(np.abs(out.cpu().numpy()[0] - o_ref).max())
    assert err <= H.OUT_ATOL, err
    # every rank holds the same joined output
    for _, b, _ in shards:
        assert torch.equal(b.out, out)


def test_split_equals_one_gpu_step():
    """The joined output against ts_decode_step on the whole sequence (one
    GPU, same inputs): same selection, outputs within the attention
    tolerance (the normalisers are combined in another order)."""
    (n, h_q, h_kv, d, k, s, l, lens), kk, vv, q, shards, out = _run("qwen_shape_uneven_four")
    m = H.ts()
    kv = m.KVCache(kk, vv, np.array([0, n]), h_q)
    buf = m.StepBuffers(kv, k, s, l)
    m.ts_decode_step(kv, q, buf.q_prev, buf.reuse, True, 2.0, k, s, l, buf.votes, buf.ids, buf.count, buf.out,
                     buf.ws, buf.cos)
    torch.cuda.synchronize()
    c = int(buf.count.cpu().numpy()[0])
    one = buf.ids.cpu().numpy()[0][:c]
    union = sorted(int(x) + t for kv_, b, t in shards for x in b.step.ids.cpu().numpy()[0][:int(b.step.count[0])])
    votes = np.concatenate([b.step.votes.cpu().numpy()[:kv_.n_total] for kv_, b, _ in shards])
    diff = set(one.tolist()) ^ set(union)
    if diff:   # only ties at the threshold may differ (votes rounded in another order)
        v1 = buf.votes.cpu().numpy()
        thr = np.sort(v1[s:n - l])[::-1][k - 1]
        assert all(abs(v1[i] - thr) <= 1e-6 * thr for i in diff), diff
    assert np.allclose(votes, buf.votes.cpu().numpy()[:n], rtol=1e-5, atol=1e-30)
    assert float((out - buf.out).abs().max()) <= H.OUT_ATOL


def test_normalisers_of_a_batch_with_reuse_and_an_empty_sequence():
    """ts_score_normalisers on a batch of several sequences: the merge writes
    every fresh, nonempty sequence's per-head log-normalisers straight into
    L_out (against the oracle's, 1e-4 absolute: a vote's relative error is
    about the normaliser's absolute one), and leaves the rows of the
    sequence that reuses and of the empty one as they were."""
    lengths, h_q, h_kv, d = [2000, 0, 1500, 700], 28, 4, 128
    off = W.seq_offsets(lengths)
    kk, vv = W.random_kv(int(off[-1]), h_kv, d, 21, device="cuda")
    q = torch.randn((len(lengths), h_q, d), generator=torch.Generator().manual_seed(22)).to(torch.bfloat16).cuda()
    m = H.ts()
    kv = m.KVCache(kk, vv, off, h_q)
    buf = m.StepBuffers(kv, 64, 4, 16)
    reuse = torch.tensor([0, 0, 1, 0], dtype=torch.int32, device="cuda")
    L_out = torch.full((len(lengths) * h_q,), 123.0, dtype=torch.float64, device="cuda")
    m.ts_score_normalisers(kv, q, reuse, L_out, buf.ws)
    torch.cuda.synchronize()
    got = L_out.cpu().numpy().reshape(len(lengths), h_q)
    kb, qb = W.bf16_bits(kk), W.bf16_bits(q)
    for b, n in enumerate(lengths):
        if n == 0 or b == 2:
            assert np.all(got[b] == 123.0), b
            continue
        _, L_ref = oracle.votes(kb[int(off[b]):int(off[b + 1])], qb[b])
        assert np.abs(got[b] - L_ref).max() <= 1e-4, (b, np.abs(got[b] - L_ref).max())


def test_split_rank_with_nothing_selected():
    """A middle shard whose keys are all zero (logits 0, below the other
    shards' top votes), outside the sink and local windows: its rank selects
    no token at all (count 0, log-sum-exp -inf), and the join leaves it out;
    the joined selection and output still follow the oracle."""
    n, h_q, h_kv, d, k, s, l = 3000, 8, 2, 128, 16, 4, 16
    lens = [1000, 1000, 1000]
    kk, vv = W.random_kv(n, h_kv, d, 31, device="cuda")
    kk[1000:2000] = 0
    q = torch.randn((1, h_q, d), generator=torch.Generator().manual_seed(32)).to(torch.bfloat16).cuda()
    m = H.ts()
    from query_aware_kv_ts_b200 import split
    shards, t = [], 0
    for ln in lens:
        kv = m.KVCache(kk[t:t + ln], vv[t:t + ln], np.array([0, ln]), h_q)
        shards.append((kv, split.ShardBuffers(kv, k, s, l, len(lens)), t))
        t += ln
    out = split.emulate_split_decode_step(shards, q, n)
    torch.cuda.synchronize()
    assert int(shards[1][1].step.count.cpu()[0]) == 0
    assert torch.isinf(shards[1][1].lse).all() and (shards[1][1].lse < 0).all()
    kb, vb, qb = W.bf16_bits(kk), W.bf16_bits(vv), W.bf16_bits(q)[0]
    votes = np.concatenate([b.step.votes.cpu().numpy()[:kv.n_total] for kv, b, _ in shards])
    union = np.array(sorted(int(x) + t for kv, b, t in shards
                            for x in b.step.ids.cpu().numpy()[0][:int(b.step.count.cpu()[0])]), np.int32)
    want, m_ = oracle.select(votes.astype(np.float64), k, s, l)
    assert union.size == m_ and np.array_equal(union, want[:m_])
    o_ref = oracle.sparse_attn(kb, vb, qb, union, union.size)
    assert float(np.abs(out.cpu().numpy()[0] - o_ref).max()) <= H.OUT_ATOL
