"""GPU parity: the C-ABI decode step against the float64 oracle.

Small synthetic cases cover every kernel specialisation (head_dim 64/128,
group sizes 1..16, h_kv 1..8), ragged batches with empty and one-token
sequences, tails that are not a multiple of the tile, windows larger than the
sequence, k = 0 and k >= candidates, tied votes, padded strides, very peaked
scores, more than 32 sequences, and the largest batch (1024) and selection
capacity (16384) the library takes.  Each case spans several tiles and a
ragged tail."""
import zlib

import numpy as np
import pytest
import torch

import gpu_helpers as H
import workloads as W

pytestmark = pytest.mark.gpu


def _case(lengths, h_q, h_kv, d, seed, dist="normal", strides=None, scale=0.0, planted=0):
    off = W.seq_offsets(lengths)
    n = int(off[-1])
    st, sh = strides if strides else (None, None)
    k, v = W.random_kv(n, h_kv, d, seed, device="cuda", dist=dist, stride_tok=st, stride_head=sh)
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn((len(lengths), h_q, d), generator=g).to(torch.bfloat16)
    if planted:
        G = h_q // h_kv
        for b in range(len(lengths)):
            nb = int(lengths[b])
            if nb == 0:
                continue
            pos = np.random.default_rng(seed + b).choice(nb, size=min(planted, nb), replace=False)
            qm = q[b].double().reshape(h_kv, G, d).mean(1)
            key = (3 * d ** 0.5 * qm / qm.norm(dim=1, keepdim=True)).to(torch.bfloat16).cuda()
            for p_ in pos:
                k[int(off[b]) + int(p_)] = key
    return H.Case(k, v, off, q.cuda(), scale=scale)


CASES = {
    # name: (lengths, h_q, h_kv, d, k, sink, local, extra)
    "d64_g2": ([4096], 4, 2, 64, 256, 4, 64, {"planted": 16}),
    "d128_g7_ragged_tail": ([1000, 37, 3333], 28, 4, 128, 100, 4, 50, {"planted": 8}),
    "g8_hkv8": ([777], 64, 8, 128, 64, 2, 16, {}),
    "g16_two_ntiles": ([2048, 513], 32, 2, 128, 128, 4, 32, {}),
    "g16_d64": ([999], 16, 1, 64, 90, 3, 7, {}),
    "mha_g1": ([500], 4, 4, 64, 50, 1, 10, {}),
    "hkv1_d128": ([1500], 8, 1, 128, 100, 4, 100, {}),
    "short_sequences": ([3, 10, 70, 1], 28, 4, 128, 16, 4, 64, {}),
    "k_above_candidates": ([300], 4, 2, 64, 1000, 4, 64, {}),
    "k_zero": ([300], 4, 2, 64, 0, 4, 64, {}),
    "empty_sequences": ([0, 500, 0, 1], 4, 2, 64, 32, 4, 8, {}),
    "no_windows": ([1234], 8, 2, 128, 77, 0, 0, {}),
    "constant_keys_all_tied": ([1000], 4, 2, 64, 100, 4, 16, {"dist": "const"}),
    "integer_keys_many_ties": ([2000], 28, 4, 128, 200, 4, 64, {"dist": "int"}),
    "padded_strides": ([3000], 28, 4, 128, 256, 4, 64, {"strides": (4 * 128 * 2 + 64, 256)}),
    "peaked_scores": ([2500], 8, 2, 128, 64, 4, 32, {"scale": 1.0}),
    "d64_hkv8_g2": ([1500, 77], 16, 8, 64, 100, 4, 32, {"planted": 8}),
    # more than 32 sequences (score pass A's general chunk-table path)
    "batch_40_qwen_heads": ([int(x) for x in np.random.default_rng(40).integers(1, 700, 40)], 28, 4, 128, 64, 4,
                            32, {}),
    # the largest batch and the largest selection the library takes
    "max_batch_1024": ([int(x) for x in np.random.default_rng(1024).integers(0, 41, 1024)], 4, 2, 64, 8, 2, 4, {}),
    "max_capacity_16384": ([20000], 4, 2, 64, 16384 - 4 - 64, 4, 64, {"planted": 32}),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_case(name):
    lengths, h_q, h_kv, d, k, s, l, extra = CASES[name]
    case = _case(lengths, h_q, h_kv, d, seed=zlib.crc32(name.encode()) % 10000, **extra)
    buf = H.run_step(case, k, s, l)
    H.check_step(case, buf, k, s, l)


def test_all_tied_picks_lowest_ids():
    case = _case([1000], 4, 2, 64, 3, dist="const")
    buf = H.run_step(case, 100, 4, 16)
    ids = buf.ids.cpu().numpy()[0]
    want = list(range(0, 4)) + list(range(4, 104)) + list(range(984, 1000))
    assert ids[:buf.count.item()].tolist() == want


def test_deterministic():
    case = _case([5000, 777], 28, 4, 128, 11, planted=5)
    a = H.run_step(case, 300, 4, 64)
    va, ia, oa = a.votes.clone(), a.ids.clone(), a.out.clone()
    for _ in range(3):
        b = H.run_step(case, 300, 4, 64, buf=a)
        assert torch.equal(va, b.votes) and torch.equal(ia, b.ids) and torch.equal(oa, b.out)


def test_planted_keys_selected():
    case = _case([8192], 28, 4, 128, 5, planted=40)
    buf = H.run_step(case, 64, 4, 64)
    ids = set(buf.ids.cpu().numpy()[0].tolist())
    # the 40 planted keys carry the top votes
    votes = buf.votes.cpu().numpy()
    top = np.argsort(-votes)[:40]
    assert set(top.tolist()) <= ids


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_score_matches_oracle_and_two_phase(name):
    """ts_score_fused (logits, normalisers and votes in one kernel, a few kv
    heads per pass) against the oracle's votes, and against ts_score (the
    two-phase scoring) to within their two roundings; a second call on the
    same workspace gives the same votes (the kernel's grid-barrier counters
    return to zero)."""
    lengths, h_q, h_kv, d, k, s, l, extra = CASES[name]
    case = _case(lengths, h_q, h_kv, d, seed=zlib.crc32(name.encode()) % 10000, **extra)
    m = H.ts()
    buf = m.StepBuffers(case.kv, k, s, l)
    m.ts_score(case.kv, case.q, None, buf.votes, buf.ws)
    two = buf.votes.cpu().numpy().copy()
    m.ts_score_fused(case.kv, case.q, None, buf.votes, buf.ws)
    fused = buf.votes.cpu().numpy().copy()
    m.ts_score_fused(case.kv, case.q, None, buf.votes, buf.ws)
    assert np.array_equal(buf.votes.cpu().numpy().view(np.uint32), fused.view(np.uint32))
    status, site = m.ts_get_device_status(buf.ws)
    assert status == m.TS_OK, (status, site)
    qb = W.bf16_bits(case.q)
    for b in range(case.B):
        lo, hi = case.seq(b)
        if hi == lo:
            continue
        v_ref, _ = H.oracle.votes(case.kb[lo:hi], qb[b], case.oracle_scale())
        H.check_votes(two[lo:hi], v_ref, h_q)
        H.check_votes(fused[lo:hi], v_ref, h_q)
        rel = np.abs(two[lo:hi].astype(np.float64) - fused[lo:hi]) / np.maximum(v_ref, 1e-30)
        assert rel.max() < 1e-5, rel.max()


@pytest.mark.parametrize("cfg_name", ["qwen7b_32k", "llama8b_b4", "ragged_b32", "qwen7b_1m"])
def test_fused_score_full_size(cfg_name):
    """ts_score_fused at the workloads' full sizes (one pass at 32K; two at
    4 x 131072; one kv head per pass at 32 ragged sequences and at 1M tokens)
    against the oracle's votes, sequence by sequence."""
    cfg = W.CONFIGS[cfg_name]
    case, _ = H.config_case(cfg)
    m = H.ts()
    buf = m.StepBuffers(case.kv, cfg.k, cfg.n_sink, cfg.n_local)
    m.ts_score_fused(case.kv, case.q, None, buf.votes, buf.ws)
    votes = buf.votes.cpu().numpy()
    qb = W.bf16_bits(case.q)
    for b in range(case.B):
        lo, hi = case.seq(b)
        v_ref, _ = H.oracle.votes(case.kb[lo:hi], qb[b], case.oracle_scale())
        H.check_votes(votes[lo:hi], v_ref, cfg.h_q)


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_on_cuda_cores(name, monkeypatch):
    """The CUDA-core (fp32 FMA) variant of the sparse attention, selected with
    TS_ATTN_CUDA_CORES=1, against the oracle's attention over the same ids."""
    lengths, h_q, h_kv, d, k, s, l, extra = CASES[name]
    case = _case(lengths, h_q, h_kv, d, seed=zlib.crc32(name.encode()) % 10000, **extra)
    buf = H.run_step(case, k, s, l)
    tc_out = buf.out.clone()
    monkeypatch.setenv("TS_ATTN_CUDA_CORES", "1")
    H.ts().ts_sparse_attn(case.kv, case.q, buf.ids, buf.count, buf.out, buf.ws)
    torch.cuda.synchronize()
    H.check_step(case, buf, k, s, l)
    assert (buf.out - tc_out).abs().max().item() <= 2 * H.OUT_ATOL
