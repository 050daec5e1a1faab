"""Token-axis split of one long sequence across ranks (one process per GPU).

Rank r holds the contiguous shard [t_r, t_r + n_r) of the sequence's K and V
as a batch-1 cache of its own and runs the decode step's phases on it; three
small all-gathers join the shards into exactly the single-sequence step:

  1. each head's log-normaliser over the shard -> all ranks' -> their
     log-sum-exp is the sequence's (the soft vote's per-head softmax is over
     every cached token: TokenSelect README, "Key Takeaways");
  2. each shard's best k candidates as (vote, sequence id) keys -> all
     ranks' -> the k-th largest is the sequence's top-k threshold (ties to the
     lower id), and each rank keeps its own candidates at or above it, with
     its parts of the sequence's sink and local windows;
  3. each rank's attention over its selected tokens, with each head's
     log-sum-exp -> all ranks' -> the weighted combination is the attention
     over every selected token.

Every arithmetic step runs in the library's kernels (C ABI); this module only
allocates the buffers and moves them between ranks with torch.distributed
(NCCL over NVLink on GPUs).  `split_decode_step` is the per-rank SPMD step;
`emulate_split_decode_step` runs the same phases for several shards in one
process, with the all-gathers done as copies, for a single device.
"""
from __future__ import annotations

import torch

from . import (KVCache, StepBuffers, ts_merge_attention, ts_merge_normalisers, ts_score_normalisers,
               ts_score_vote_normalised, ts_select_candidates, ts_select_merge, ts_sparse_attn_lse)


class LibraryOps:
    """The phases' C-ABI calls (the default implementation of the ops)."""
    score_normalisers = staticmethod(ts_score_normalisers)
    score_vote_normalised = staticmethod(ts_score_vote_normalised)
    merge_normalisers = staticmethod(ts_merge_normalisers)
    select_candidates = staticmethod(ts_select_candidates)
    select_merge = staticmethod(ts_select_merge)
    sparse_attn_lse = staticmethod(ts_sparse_attn_lse)
    merge_attention = staticmethod(ts_merge_attention)


class ShardBuffers:
    """One rank's buffers for a split step over `parts` ranks: the shard's
    step buffers (workspace, votes, ids, count) and the joins' local and
    gathered tensors."""

    def __init__(self, kv: KVCache, k: int, n_sink: int, n_local: int, parts: int, device=None, step=None):
        dev = kv.k.device if device is None else device
        self.k, self.n_sink, self.n_local, self.parts = k, n_sink, n_local, parts
        # step: the shard's step buffers (ws, votes, ids, count), by default
        # the library's for this cache
        self.step = StepBuffers(kv, k, n_sink, n_local) if step is None else step
        rows = kv.batch * kv.h_q
        self.rows = rows
        self.L_local = torch.empty(rows, dtype=torch.float64, device=dev)
        self.L_parts = torch.empty((parts, rows), dtype=torch.float64, device=dev)
        self.L = torch.empty(rows, dtype=torch.float64, device=dev)
        self.keys = torch.empty(k, dtype=torch.int64, device=dev)          # uint64 keys, stored as int64
        self.keys_all = torch.empty((parts, k), dtype=torch.int64, device=dev)
        self.out_local = torch.empty((kv.batch, kv.h_q, kv.head_dim), dtype=torch.float32, device=dev)
        self.lse = torch.empty(rows, dtype=torch.float32, device=dev)
        self.out_parts = torch.empty((parts, kv.batch, kv.h_q, kv.head_dim), dtype=torch.float32, device=dev)
        self.lse_parts = torch.empty((parts, rows), dtype=torch.float32, device=dev)
        self.out = torch.empty((kv.batch, kv.h_q, kv.head_dim), dtype=torch.float32, device=dev)


def phase_normalisers(kv, q, buf: ShardBuffers, ops=LibraryOps):
    ops.score_normalisers(kv, q, None, buf.L_local, buf.step.ws)


def phase_votes(kv, buf: ShardBuffers, ops=LibraryOps):
    ops.merge_normalisers(buf.L_parts, buf.parts, buf.L)
    ops.score_vote_normalised(kv, None, buf.L, buf.step.votes, buf.step.ws)


def phase_candidates(kv, buf: ShardBuffers, shard_offset: int, n_global: int, ops=LibraryOps):
    ops.select_candidates(kv, buf.step.votes, buf.k, buf.n_sink, buf.n_local, shard_offset, n_global,
                          buf.step.ids, buf.step.count, buf.keys, buf.step.ws)


def phase_select_and_attend(kv, q, buf: ShardBuffers, rank: int, shard_offset: int, n_global: int,
                            ops=LibraryOps):
    ops.select_merge(kv, buf.keys_all, buf.parts, rank, buf.k, buf.n_sink, buf.n_local, shard_offset, n_global,
                     buf.step.ids, buf.step.count)
    ops.sparse_attn_lse(kv, q, buf.step.ids, buf.step.count, buf.out_local, buf.lse, buf.step.ws)


def phase_join_attention(buf: ShardBuffers, ops=LibraryOps):
    ops.merge_attention(buf.out_parts, buf.lse_parts, buf.parts, buf.out)


def _all_gather(parts: torch.Tensor, local: torch.Tensor, group):
    import torch.distributed as dist
    dist.all_gather(list(parts.unbind(0)), local.reshape(parts.shape[1:]), group=group)


def split_decode_step(kv, q, buf: ShardBuffers, shard_offset: int, n_global: int, group=None, ops=LibraryOps):
    """One decode step of the sequence, this rank's part (SPMD: every rank of
    `group` calls it with its own shard, in the same order).  Returns the
    attention output over every selected token, the same on every rank."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    assert dist.get_world_size(group) == buf.parts
    phase_normalisers(kv, q, buf, ops)
    _all_gather(buf.L_parts, buf.L_local, group)
    phase_votes(kv, buf, ops)
    phase_candidates(kv, buf, shard_offset, n_global, ops)
    _all_gather(buf.keys_all, buf.keys, group)
    phase_select_and_attend(kv, q, buf, rank, shard_offset, n_global, ops)
    _all_gather(buf.out_parts, buf.out_local, group)
    _all_gather(buf.lse_parts, buf.lse, group)
    phase_join_attention(buf, ops)
    return buf.out


def emulate_split_decode_step(shards, q, n_global: int, ops=LibraryOps):
    """The same phases for every shard in one process: shards is a list of
    (kv, ShardBuffers, shard_offset) in rank order; each all-gather is a copy
    of every shard's local tensor into every shard's gathered one.  Returns
    rank 0's output (every rank's is the same)."""
    def gather(local_of, parts_of):
        for _, b, _ in shards:
            for r, (_, src, _) in enumerate(shards):
                parts_of(b)[r].copy_(local_of(src).reshape(parts_of(b).shape[1:]))

    for kv, b, _ in shards:
        phase_normalisers(kv, q, b, ops)
    gather(lambda b: b.L_local, lambda b: b.L_parts)
    for kv, b, t in shards:
        phase_votes(kv, b, ops)
        phase_candidates(kv, b, t, n_global, ops)
    gather(lambda b: b.keys, lambda b: b.keys_all)
    for r, (kv, b, t) in enumerate(shards):
        phase_select_and_attend(kv, q, b, r, t, n_global, ops)
    gather(lambda b: b.out_local, lambda b: b.out_parts)
    gather(lambda b: b.lse, lambda b: b.lse_parts)
    for _, b, _ in shards:
        phase_join_attention(b, ops)
    return shards[0][1].out
