"""Paged KV caches (a block table into a pool of pages) against the packed
layout and the oracle.

Each case builds its sequences' K and V as a packed cache, then scatters the
same rows page by page into a pool half again as large, in a random page
order, with junk (large values) in the pool's unused pages and -1 in the block
table's unused entries.  The decode step on the paged cache must give exactly
(bit for bit) what it gives on the packed cache (the kernels take the same
chunks in the same order; only the rows' addresses differ), and so follow the
oracle; with pages shorter than a scoring chunk (and at least 16 tokens) the
scoring stage holds its rows page by page, and the results follow the oracle
and match the packed ones up to the normalisers' rounding."""
import numpy as np
import pytest
import torch

import gpu_helpers as H
import workloads as W

pytestmark = pytest.mark.gpu


def _paged(k, v, off, page, seed, extra=0.5):
    """Pool of pages holding the packed rows k, v [sum_n, h_kv, d] of the
    sequences at off, and the block table [B, stride] (int32, -1 unused)."""
    lengths = np.diff(off)
    pages = [int(-(-n // page)) for n in lengths]
    stride = max(1, max(pages))
    used = sum(pages)
    pool_pages = used + int(extra * used) + 1
    rng = np.random.default_rng(seed)
    phys = rng.permutation(pool_pages)[:used]
    h_kv, d = k.shape[1], k.shape[2]
    kp = torch.full((pool_pages * page, h_kv, d), 1.0e4, dtype=torch.bfloat16, device=k.device)
    vp = torch.full((pool_pages * page, h_kv, d), -1.0e4, dtype=torch.bfloat16, device=k.device)
    table = np.full((len(lengths), stride), -1, np.int32)
    j = 0
    for b, n in enumerate(lengths):
        for pg in range(pages[b]):
            lo = int(off[b]) + pg * page
            hi = min(int(off[b + 1]), lo + page)
            r0 = int(phys[j]) * page
            kp[r0:r0 + hi - lo] = k[lo:hi]
            vp[r0:r0 + hi - lo] = v[lo:hi]
            table[b, pg] = int(phys[j])
            j += 1
    return kp, vp, torch.from_numpy(table).cuda()


CASES = {
    # name: (lengths, h_q, h_kv, d, k, sink, local, page)
    "qwen_shape_page32": ([5000], 28, 4, 128, 512, 4, 128, 32),
    "qwen_shape_page256_ragged": ([3000, 77, 4100], 28, 4, 128, 300, 4, 64, 256),
    "llama_shape_page16_b4": ([2048, 1500, 999, 3], 32, 8, 128, 256, 4, 64, 16),
    "tiny_shape_page64": ([4096], 4, 2, 64, 256, 4, 64, 64),
    "hkv1_page128": ([1500, 600], 8, 1, 128, 100, 4, 32, 128),
    "g16_page4096": ([5000], 32, 2, 128, 128, 4, 32, 4096),
    "empty_and_short_page64": ([0, 500, 0, 3], 4, 2, 64, 32, 4, 8, 64),
    # pages shorter than a scoring chunk of 128/h_kv tokens: one box per page
    # (every kv head), or per page and kv head for 8-token pages
    "qwen_shape_page16_ragged": ([5000, 33, 1], 28, 4, 128, 512, 4, 128, 16),
    "tiny_shape_page16": ([4096, 70], 4, 2, 64, 256, 4, 64, 16),
    "tiny_shape_page32": ([3000], 4, 2, 64, 128, 4, 64, 32),
    "g16_hkv2_page16": ([2048, 513], 32, 2, 128, 128, 4, 32, 16),
    "hkv1_page8": ([1500, 600], 8, 1, 128, 100, 4, 32, 8),
    "g16_hkv2_page8_d64": ([999], 32, 2, 64, 90, 3, 7, 8),
}


def _page_major(page, h_kv):
    """Pages of 16 or more tokens but shorter than a scoring chunk of
    128 / h_kv tokens are loaded one box of every kv head per page."""
    return h_kv > 1 and 16 <= page < 128 // h_kv


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("fused", [False, True])
def test_paged_equals_packed(name, fused):
    lengths, h_q, h_kv, d, k_top, s, l, page = CASES[name]
    off = W.seq_offsets(lengths)
    k, v = W.random_kv(int(off[-1]), h_kv, d, 77 + page, device="cuda")
    q = torch.randn((len(lengths), h_q, d), generator=torch.Generator().manual_seed(page)).to(torch.bfloat16).cuda()
    packed = H.Case(k, v, off, q)
    kp, vp, table = _paged(k, v, off, page, seed=page)
    m = H.ts()
    paged_kv = m.KVCache(kp, vp, off, h_q, page_table=table, page_size=page)
    if fused:
        bp = m.StepBuffers(packed.kv, k_top, s, l)
        bq = m.StepBuffers(paged_kv, k_top, s, l)
        for kv_, b_ in ((packed.kv, bp), (paged_kv, bq)):
            m.ts_decode_step(kv_, q, b_.q_prev, b_.reuse, True, 2.0, k_top, s, l, b_.votes, b_.ids, b_.count,
                             b_.out, b_.ws, b_.cos)
        torch.cuda.synchronize()
    else:
        bp = H.run_step(packed, k_top, s, l)
        paged = H.Case(kp, vp, off, q)
        paged.kv = paged_kv
        bq = H.run_step(paged, k_top, s, l)
    if _page_major(page, h_kv):
        # the stage's rows go page by page, so the epilogue's per-warp
        # (max, sum) partials cover other token sets than in the packed
        # layout: the normalisers, and through them the votes, may differ in
        # the last bits; both follow the oracle
        vp_, vq_ = bp.votes.cpu().numpy().astype(np.float64), bq.votes.cpu().numpy().astype(np.float64)
        assert np.allclose(vq_, vp_, rtol=1e-5, atol=1e-30)
        H.check_step(packed, bp, k_top, s, l)
    else:
        for n_ in ("votes", "ids", "count", "out"):
            a_, b_ = getattr(bp, n_).cpu().numpy(), getattr(bq, n_).cpu().numpy()
            assert np.array_equal(a_.view(np.uint8), b_.view(np.uint8)), n_
    H.check_step(packed, bq, k_top, s, l)
    status, site = m.ts_get_device_status(bq.ws)
    assert status == m.TS_OK, (status, site)


def test_paged_noalloc_attention():
    lengths, h_q, h_kv, d, k_top, s, l, page = CASES["llama_shape_page16_b4"]
    off = W.seq_offsets(lengths)
    k, v = W.random_kv(int(off[-1]), h_kv, d, 5, device="cuda")
    q = torch.randn((len(lengths), h_q, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    packed = H.Case(k, v, off, q)
    bp = H.run_step(packed, k_top, s, l)
    kp, vp, table = _paged(k, v, off, page, seed=9)
    m = H.ts()
    paged_kv = m.KVCache(kp, vp, off, h_q, page_table=table, page_size=page)
    out = torch.full_like(bp.out, float("nan"))
    m.ts_sparse_attn_noalloc(paged_kv, q, bp.ids, bp.count, out)
    torch.cuda.synchronize()
    assert torch.equal(out, bp.out)


def test_paged_unsupported_shapes():
    m = H.ts()
    off = W.seq_offsets([100])
    k, v = W.random_kv(128, 4, 128, 1, device="cuda")
    table = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    q = torch.zeros((1, 28, 128), dtype=torch.bfloat16, device="cuda")
    # page sizes below 8 tokens (one swizzle atom of a TMA box) are not taken
    kv = m.KVCache(k, v, off, 28, page_table=torch.zeros((1, 32), dtype=torch.int32, device="cuda"), page_size=4)
    with pytest.raises(m.TsError, match="page_size"):
        m.ts_workspace_bytes(kv, 16, 4, 16)
    # the fused scoring takes packed caches only
    kv = m.KVCache(k, v, off, 28, page_table=table, page_size=32)
    ws = torch.zeros(m.ts_workspace_bytes(kv, 16, 4, 16), dtype=torch.uint8, device="cuda")
    votes = torch.zeros(100, dtype=torch.float32, device="cuda")
    with pytest.raises(m.TsError) as e:
        m.ts_score_fused(kv, q, None, votes, ws)
    assert e.value.status == m.TS_ERR_UNSUPPORTED
