"""ts_sparse_attn_noalloc: attention for callers that cannot allocate.

Some hosts own all device memory through their own pool and let no library
allocate or take a workspace after start-up.  ts_sparse_attn_noalloc serves
them with its scratch in a fixed array inside libts.  These tests call it
through the C ABI twice in a row (two different shapes, so the second call
runs on whatever the first left in the shared array) and compare each output
with the workspace-based ts_sparse_attn, within the attention tolerance of the
parity tests.  They pass alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

import gpu_helpers as H
import workloads as W

pytestmark = pytest.mark.gpu


def _case(lengths, h_q, h_kv, d, k, s, l, seed):
    off = W.seq_offsets(lengths)
    kk, vv = W.random_kv(int(off[-1]), h_kv, d, seed, device="cuda")
    q = torch.randn((len(lengths), h_q, d), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    case = H.Case(kk, vv, off, q.cuda())
    buf = H.run_step(case, k, s, l)          # ids/count from the normal path; out from ts_sparse_attn
    return case, buf


def test_noalloc_matches_workspace_attention_two_calls():
    m = H.ts()
    first = _case([32768], 28, 4, 128, 2048, 4, 512, seed=7)
    second = _case([3000, 17, 9000], 32, 8, 64, 256, 4, 64, seed=8)
    outs = []
    for case, buf in (first, second):
        out = torch.full_like(buf.out, float("nan"))
        m.ts_sparse_attn_noalloc(case.kv, case.q, buf.ids, buf.count, out)
        torch.cuda.synchronize()
        ref = buf.out
        err = (out - ref).abs().max().item()
        assert err <= H.OUT_ATOL, err
        outs.append(out.clone())
    # and once more on the first shape after the second one used the array
    case, buf = first
    out = torch.empty_like(buf.out)
    m.ts_sparse_attn_noalloc(case.kv, case.q, buf.ids, buf.count, out)
    torch.cuda.synchronize()
    assert (out - buf.out).abs().max().item() <= H.OUT_ATOL
    assert torch.equal(out, outs[0])


def test_noalloc_rejects_oversize_shapes():
    m = H.ts()
    # 1024 sequences x 8 kv heads x 16 heads per group: the split-K partials
    # alone exceed the fixed 4 MiB scratch
    lengths = [64] * 1024
    off = W.seq_offsets(lengths)
    kk, vv = W.random_kv(int(off[-1]), 8, 128, 3, device="cuda")
    q = torch.zeros((1024, 128, 128), dtype=torch.bfloat16, device="cuda")
    kv = m.KVCache(kk, vv, off, 128)
    ids = torch.zeros((1024, 64), dtype=torch.int32, device="cuda")
    count = torch.zeros(1024, dtype=torch.int32, device="cuda")
    out = torch.zeros((1024, 128, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(m.TsError) as e:
        m.ts_sparse_attn_noalloc(kv, q, ids, count, out)
    assert e.value.status == m.TS_ERR_UNSUPPORTED
    assert "4194304" in str(e.value)


def _scratch_bytes(B, h_kv, G, d, cap):
    # split-K partials: one (d + 4)-float row per (sequence, kv head, split, head)
    return B * h_kv * -(-cap // 64) * G * (d + 4) * 4


def test_noalloc_scratch_limit_boundary():
    """Either side of the 4 MiB limit, through the C ABI: 2 sequences, one kv
    head of 16 query heads, d = 128; an ids row of 15872 needs 248 splits
    (4,190,208 bytes: accepted, and equal to the workspace attention), one more
    id needs 249 (4,207,104 bytes: rejected before anything is launched)."""
    m = H.ts()
    limit = 4 << 20
    assert _scratch_bytes(2, 1, 16, 128, 15872) <= limit < _scratch_bytes(2, 1, 16, 128, 15873)
    case, buf = _case([20000, 16000], 16, 1, 128, 15872 - 4 - 64, 4, 64, seed=11)
    assert buf.ids.shape == (2, 15872)
    out = torch.full_like(buf.out, float("nan"))
    m.ts_sparse_attn_noalloc(case.kv, case.q, buf.ids, buf.count, out)
    torch.cuda.synchronize()
    assert (out - buf.out).abs().max().item() <= H.OUT_ATOL
    wide = torch.full((2, 15873), -1, dtype=torch.int32, device="cuda")
    wide[:, :15872] = buf.ids
    out2 = torch.full_like(buf.out, float("nan"))
    with pytest.raises(m.TsError) as e:
        m.ts_sparse_attn_noalloc(case.kv, case.q, wide, buf.count, out2)
    assert e.value.status == m.TS_ERR_UNSUPPORTED
    assert str(_scratch_bytes(2, 1, 16, 128, 15873)) in str(e.value)
    torch.cuda.synchronize()
    assert torch.isnan(out2).all(), "a rejected call must not launch"
