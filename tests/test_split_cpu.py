"""The token-axis split's choreography on CPU (gloo, world sizes 2 and 3):
every rank holds one shard of a sequence and runs
query_aware_kv_ts_b200.split.split_decode_step, whose three all-gathers go
through torch.distributed; the phases' arithmetic is done here by stand-ins
written from the oracle (no GPU), so what is checked is the order of the
phases and exchanges, the shard offsets and windows, and the ranks' indexing
of the gathered tensors: the joined output must be the oracle's attention
over the whole sequence's selection, on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _bits_f64(u16):
    return (np.asarray(u16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class OracleOps:
    """The phases' arithmetic, from the oracle's definitions, on CPU tensors."""

    def __init__(self):
        self.logits = {}

    def score_normalisers(self, kv, q, reuse, L_out, ws):
        import oracle
        import workloads as W
        kb, qb = W.bf16_bits(kv.k), W.bf16_bits(q)[0]
        h_q = qb.shape[0]
        s = np.stack([oracle.head_logits(kb, qb, h) for h in range(h_q)]) if kb.shape[0] else np.zeros((h_q, 0))
        self.logits[id(ws)] = s
        L = np.array([oracle.softmax_row(s[h])[1] if s.shape[1] else -np.inf for h in range(h_q)])
        L_out.copy_(torch.from_numpy(L))

    def merge_normalisers(self, L_parts, parts, L_out):
        P = L_parts.numpy()
        M = P.max(axis=0)
        with np.errstate(invalid="ignore"):
            L = np.where(np.isneginf(M), -np.inf, M + np.log(np.exp(P - M).sum(axis=0)))
        L_out.copy_(torch.from_numpy(L))

    def score_vote_normalised(self, kv, reuse, L_in, votes, ws):
        s = self.logits[id(ws)]
        v = np.exp(s - L_in.numpy()[:, None]).sum(axis=0) if s.shape[1] else np.zeros(0)
        votes[:v.size] = torch.from_numpy(v.astype(np.float32))

    @staticmethod
    def _windows(n_loc, n_sink, n_local, t, n_global):
        s = min(n_sink, n_global)
        l0 = max(n_global - n_local, s)
        return max(0, min(s, t + n_loc) - t), max(0, t + n_loc - max(l0, t))

    def select_candidates(self, kv, votes, k, n_sink, n_local, t, n_global, ids, count, keys, ws):
        import oracle
        n_loc = kv.n_total
        s_loc, l_loc = self._windows(n_loc, n_sink, n_local, t, n_global)
        v = votes.numpy()[:n_loc].astype(np.float64)
        row, m = oracle.select(v, k, s_loc, l_loc)
        top = row[s_loc:m - l_loc]
        vb = votes.numpy()[:n_loc].view(np.uint32)
        out = np.zeros(k, np.uint64)
        out[:top.size] = (vb[top].astype(np.uint64) << np.uint64(32)) | \
            (np.uint64(0xffffffff) - (top.astype(np.uint64) + np.uint64(t)))
        keys.copy_(torch.from_numpy(out.view(np.int64)))

    def select_merge(self, kv, keys_all, parts, rank, k, n_sink, n_local, t, n_global, ids, count):
        n_loc = kv.n_total
        s_loc, l_loc = self._windows(n_loc, n_sink, n_local, t, n_global)
        allk = keys_all.numpy().view(np.uint64).reshape(-1)
        real = np.sort(allk[allk != 0])[::-1]
        T = real[k - 1] if real.size > k else (real[-1] if real.size else np.uint64(1))
        own = keys_all.numpy().view(np.uint64)[rank]
        chosen = [int(np.uint64(0xffffffff) - (x & np.uint64(0xffffffff))) - t for x in own if x != 0 and x >= T]
        row = list(range(s_loc)) + chosen + list(range(n_loc - l_loc, n_loc))
        cap = ids.numel()
        r = np.full(cap, -1, np.int32)
        r[:len(row)] = row
        ids.copy_(torch.from_numpy(r))
        count.fill_(len(row))

    def sparse_attn_lse(self, kv, q, ids, count, out, lse, ws):
        import oracle
        import workloads as W
        kb, vb, qb = W.bf16_bits(kv.k), W.bf16_bits(kv.v), W.bf16_bits(q)[0]
        m = int(count[0])
        sel = ids.numpy()[:m]
        out[0] = torch.from_numpy(oracle.sparse_attn(kb, vb, qb, sel, m).astype(np.float32))
        h_q, h_kv, d = qb.shape[0], kb.shape[1], kb.shape[2]
        G = h_q // h_kv
        L = np.full(h_q, -np.inf)
        if m:
            qf, kf = _bits_f64(qb), _bits_f64(kb[sel])
            for h in range(h_q):
                s = kf[:, h // G, :] @ qf[h] / np.sqrt(d)
                M = s.max()
                L[h] = M + np.log(np.exp(s - M).sum())
        lse.copy_(torch.from_numpy(L.astype(np.float32)))

    def merge_attention(self, out_parts, lse_parts, parts, out):
        O = out_parts.numpy().reshape(parts, -1, out.shape[-1]).astype(np.float64)
        Lp = lse_parts.numpy().astype(np.float64)
        M = Lp.max(axis=0)
        w = np.where(np.isneginf(Lp), 0.0, np.exp(Lp - np.where(np.isneginf(M), 0.0, M)))
        z = w.sum(axis=0)
        res = (w[:, :, None] * O).sum(axis=0) / np.where(z > 0, z, 1.0)[:, None]
        out.copy_(torch.from_numpy(res.astype(np.float32)).reshape(out.shape))


class CpuStep:
    def __init__(self, n_loc, k, n_sink, n_local):
        self.ws = torch.zeros(8, dtype=torch.uint8)
        self.votes = torch.zeros(max(n_loc, 1), dtype=torch.float32)
        self.ids = torch.full((k + n_sink + n_local,), -1, dtype=torch.int32)
        self.count = torch.zeros(1, dtype=torch.int32)


N, H_Q, H_KV, D, K_TOP, SINK, LOCAL = 900, 8, 2, 64, 64, 6, 40


def _inputs():
    import workloads as W
    kk, vv = W.random_kv(N, H_KV, D, 31)
    q = torch.randn((1, H_Q, D), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    return kk, vv, q


def _worker(rank, world, port, lens, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import torch.distributed as dist
    from query_aware_kv_ts_b200 import KVCache, split
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kk, vv, q = _inputs()
        t = sum(lens[:rank])
        ln = lens[rank]
        kv = KVCache(kk[t:t + ln], vv[t:t + ln], np.array([0, ln]), H_Q)
        buf = split.ShardBuffers(kv, K_TOP, SINK, LOCAL, world, device="cpu", step=CpuStep(ln, K_TOP, SINK, LOCAL))
        out = split.split_decode_step(kv, q, buf, t, N, ops=OracleOps())
        c = int(buf.step.count[0])
        q_out.put((rank, out.numpy().copy(), [int(x) + t for x in buf.step.ids.numpy()[:c]]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [[450, 450], [3, 600, 297], [850, 20, 30]])
def test_split_choreography_gloo(lens):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import oracle
    import workloads as W
    world = len(lens)
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, lens, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=240) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    kk, vv, q = _inputs()
    kb, vb, qb = W.bf16_bits(kk), W.bf16_bits(vv), W.bf16_bits(q)[0]
    v_ref, _ = oracle.votes(kb, qb)
    ids_ref, m_ref = oracle.select(v_ref, K_TOP, SINK, LOCAL)
    union = sorted(x for _, _, ids in res for x in ids)
    assert union == ids_ref[:m_ref].tolist()
    o_ref = oracle.sparse_attn(kb, vb, qb, ids_ref, m_ref)
    for _, out, _ in res:
        assert np.abs(out[0] - o_ref).max() <= 1e-4
