"""Python binding of libts, the B200 (sm_100a) TokenSelect decode-step library.

Argument marshalling only: every function here forwards torch tensors' device
pointers and the current CUDA stream to the C ABI declared in include/ts.h,
under the same names.  Every result is computed by the library's CUDA kernels;
there is no Python or CPU fallback, and importing this package fails loudly if
the compiled library is missing (build it with
``python query_aware_kv_ts_b200/csrc/build.py``).

TokenSelect (GitHub README, "Key Takeaways"): per-head Q.K criticality of every
cached token, per-head softmax over tokens summed over heads (soft vote), top-k
token selection with sink and local windows, a Selection Cache that reuses the
previous selection for similar consecutive queries, and attention over the
selected tokens only.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libts.so")

TS_OK = 0
TS_ERR_INVALID_ARG = 1
TS_ERR_UNSUPPORTED = 2
TS_ERR_WORKSPACE = 3
TS_ERR_CUDA = 4
TS_ERR_DEVICE_TIMEOUT = 5


class TsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (_status_name(status), message))
        self.status = status


class ts_kv_t(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("seq_offsets_dev", ctypes.c_void_p), ("seq_offsets_host", ctypes.c_void_p),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("stride_tok", ctypes.c_int64), ("stride_head", ctypes.c_int64),
        ("scale", ctypes.c_float),
        ("capacity", ctypes.c_int64),
        ("page_size", ctypes.c_int32), ("page_table_stride", ctypes.c_int32),
        ("pool_pages", ctypes.c_int64),
        ("page_table_dev", ctypes.c_void_p),
    ]


if not os.path.exists(LIB_PATH):
    raise ImportError("libts.so is not built at %s; run `python query_aware_kv_ts_b200/csrc/build.py`" % LIB_PATH)
_lib = ctypes.CDLL(LIB_PATH)

_P, _I32, _U32, _F64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_double, ctypes.c_size_t
_KV = ctypes.POINTER(ts_kv_t)
_SIGS = {
    "ts_workspace_bytes": (_SZ, [_KV, _I32, _I32, _I32]),
    "ts_workspace_init": (ctypes.c_int, [_P, _SZ, _P]),
    "ts_selcache": (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _F64, _P]),
    "ts_score": (ctypes.c_int, [_KV, _P, _P, _P, _P, _SZ, _P]),
    "ts_score_logits": (ctypes.c_int, [_KV, _P, _P, _P, _SZ, _P]),
    "ts_score_vote": (ctypes.c_int, [_KV, _P, _P, _P, _SZ, _P]),
    "ts_score_fused": (ctypes.c_int, [_KV, _P, _P, _P, _P, _SZ, _P]),
    "ts_select": (ctypes.c_int, [_KV, _P, _I32, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    "ts_sparse_attn": (ctypes.c_int, [_KV, _P, _P, _P, _I32, _P, _P, _SZ, _P]),
    "ts_sparse_attn_noalloc": (ctypes.c_int, [_KV, _P, _P, _P, _I32, _P, _P]),
    "ts_decode_step": (ctypes.c_int, [_KV, _P, _P, _P, _P, _I32, _F64, _I32, _I32, _I32, _P, _P, _P, _P, _P,
                                      _SZ, _P]),
    "ts_decode_step_kernels": (_I32, [_KV, _I32, _I32, _I32]),
    "ts_append_kv": (ctypes.c_int, [_KV, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "ts_get_device_status": (ctypes.c_int, [_P, _SZ, ctypes.POINTER(_U32), _P]),
    "ts_selftest_expire_wait": (ctypes.c_int, [_P, _SZ, _U32, _P]),
    "ts_score_normalisers": (ctypes.c_int, [_KV, _P, _P, _P, _P, _SZ, _P]),
    "ts_score_vote_normalised": (ctypes.c_int, [_KV, _P, _P, _P, _P, _SZ, _P]),
    "ts_merge_normalisers": (ctypes.c_int, [_P, _I32, ctypes.c_int64, _P, _P]),
    "ts_select_candidates": (ctypes.c_int, [_KV, _P, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64, _P, _P, _P,
                                            _P, _SZ, _P]),
    "ts_select_merge": (ctypes.c_int, [_KV, _P, _I32, _I32, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64, _P,
                                       _P, _P]),
    "ts_sparse_attn_lse": (ctypes.c_int, [_KV, _P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "ts_merge_attention": (ctypes.c_int, [_P, _P, _I32, ctypes.c_int64, _I32, _P, _P]),
    "ts_quest_rows": (ctypes.c_int64, [_KV, _I32]),
    "ts_quest_metadata": (ctypes.c_int, [_KV, _I32, _P, _P, _P]),
    "ts_quest_metadata_update": (ctypes.c_int, [_KV, _I32, ctypes.c_int64, _P, _P, _P]),
    "ts_quest_score": (ctypes.c_int, [_KV, _P, _I32, _P, _P, _P, _P]),
    "ts_quest_select": (ctypes.c_int, [_KV, _P, _I32, _I32, _I32, _I32, _P, _P, _P]),
    "ts_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ts_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def _status_name(s: int) -> str:
    return _lib.ts_status_string(int(s)).decode()


def _check(status: int):
    if status != TS_OK:
        raise TsError(status, _lib.ts_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("libts computes on the GPU only; got a %s tensor" % t.device)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class KVCache:
    """One layer's NHD KV cache for a (ragged) batch, described for the C ABI.

    k, v: bf16 CUDA tensors [sum_n, h_kv, d] (channel stride 1; token and head
    strides are read from the tensor); seq_offsets: int64 [B+1] (host array or
    tensor; a device copy is made once).  Keeps the ts_kv_t and the tensors it
    points at alive together.

    Paged cache: page_table (int32 [B, stride] on the device, the block table)
    and page_size; k and v are then the pool, [pool_pages * page_size, h_kv, d]."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, seq_offsets, h_q: int, scale: float = 0.0,
                 capacity: int = 0, page_table: torch.Tensor | None = None, page_size: int = 0):
        if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
            raise TypeError("K and V must be bf16")
        if k.dim() != 3 or k.shape != v.shape or k.stride() != v.stride() or k.stride(2) != 1:
            raise ValueError("K and V must be [tokens, h_kv, d] with equal strides and contiguous channels")
        off = np.ascontiguousarray(np.asarray(seq_offsets.cpu() if isinstance(seq_offsets, torch.Tensor)
                                              else seq_offsets, dtype=np.int64))
        self.k, self.v = k, v
        self.seq_offsets_host = off
        self.seq_offsets_dev = torch.from_numpy(off).to(k.device)
        self.batch = off.size - 1
        self.h_q, self.h_kv, self.head_dim = int(h_q), int(k.shape[1]), int(k.shape[2])
        stride, pool_pages, table_ptr = 0, 0, None
        if page_table is not None:
            if page_table.dtype != torch.int32 or page_table.dim() != 2 or not page_table.is_contiguous():
                raise ValueError("page_table must be a contiguous int32 [batch, stride] tensor")
            if page_size <= 0 or k.shape[0] % page_size:
                raise ValueError("page_size must divide the pool's rows")
            stride, pool_pages, table_ptr = page_table.shape[1], k.shape[0] // page_size, page_table.data_ptr()
        self.page_table = page_table
        self.struct = ts_kv_t(self.batch, self.h_q, self.h_kv, self.head_dim,
                              self.seq_offsets_dev.data_ptr(),
                              off.ctypes.data_as(ctypes.c_void_p).value,
                              k.data_ptr(), v.data_ptr(), k.stride(0), k.stride(1), float(scale),
                              int(capacity), int(page_size if page_table is not None else 0), int(stride),
                              int(pool_pages), table_ptr)
        self.capacity = int(capacity)

    @property
    def n_total(self) -> int:
        return int(self.seq_offsets_host[-1])

    def ref(self):
        return ctypes.byref(self.struct)


# ---------------------------------------------------------------------------
# The C ABI, same names
# ---------------------------------------------------------------------------

def ts_workspace_bytes(kv: KVCache, k: int, n_sink: int, n_local: int) -> int:
    n = _lib.ts_workspace_bytes(kv.ref(), k, n_sink, n_local)
    if n == 0:
        raise TsError(TS_ERR_INVALID_ARG, _lib.ts_last_error().decode())
    return int(n)


def ts_workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.ts_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ts_selcache(q, q_prev, reuse, first_step: bool, threshold: float, cos_out=None, stream=None):
    B, h_q, d = q.shape
    _check(_lib.ts_selcache(_ptr(q), _ptr(q_prev), _ptr(reuse), _ptr(cos_out), int(bool(first_step)),
                            B, h_q, d, float(threshold), _stream(stream)))


def ts_score(kv: KVCache, q, reuse, votes, ws, stream=None):
    _check(_lib.ts_score(kv.ref(), _ptr(q), _ptr(reuse), _ptr(votes), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream(stream)))


def ts_score_logits(kv: KVCache, q, reuse, ws, stream=None):
    _check(_lib.ts_score_logits(kv.ref(), _ptr(q), _ptr(reuse), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)))


def ts_score_fused(kv: KVCache, q, reuse, votes, ws, stream=None):
    """The same votes as ts_score from one cooperative kernel that scores a few
    kv heads per pass and takes each pass's votes while its logits are in L2."""
    _check(_lib.ts_score_fused(kv.ref(), _ptr(q), _ptr(reuse), _ptr(votes), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)))


def ts_score_vote(kv: KVCache, reuse, votes, ws, stream=None):
    _check(_lib.ts_score_vote(kv.ref(), _ptr(reuse), _ptr(votes), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)))


def ts_select(kv: KVCache, votes, k: int, n_sink: int, n_local: int, reuse, ids, count, ws, stream=None):
    _check(_lib.ts_select(kv.ref(), _ptr(votes), k, n_sink, n_local, _ptr(reuse), _ptr(ids), _ptr(count),
                          _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ts_sparse_attn(kv: KVCache, q, ids, count, out, ws, stream=None):
    _check(_lib.ts_sparse_attn(kv.ref(), _ptr(q), _ptr(ids), _ptr(count), ids.shape[-1], _ptr(out),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ts_sparse_attn_noalloc(kv: KVCache, q, ids, count, out, stream=None):
    """ts_sparse_attn without a workspace: for hosts that own all device memory
    and let no library allocate; the scratch is a fixed array inside libts."""
    _check(_lib.ts_sparse_attn_noalloc(kv.ref(), _ptr(q), _ptr(ids), _ptr(count), ids.shape[-1], _ptr(out),
                                       _stream(stream)))


def ts_decode_step(kv: KVCache, q, q_prev, reuse, first_step: bool, threshold: float, k: int, n_sink: int,
                   n_local: int, votes, ids, count, out, ws, cos_out=None, stream=None):
    """ts_selcache, ts_score, ts_select and ts_sparse_attn of one layer in one
    call (fewer kernels, same results)."""
    _check(_lib.ts_decode_step(kv.ref(), _ptr(q), _ptr(q_prev), _ptr(reuse), _ptr(cos_out),
                               int(bool(first_step)), float(threshold), k, n_sink, n_local, _ptr(votes),
                               _ptr(ids), _ptr(count), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream)))


def ts_append_kv(kv: KVCache, k_new, v_new, ws, stream=None):
    """Append one token ([h_kv, d] K and V rows, bf16, on the device) to a
    growing cache (KVCache(..., capacity=C), batch 1) on the device: rows at
    position n = seq_offsets[1], then seq_offsets[1] = n + 1 (device copy
    only; kv.seq_offsets_host is left as it was)."""
    _check(_lib.ts_append_kv(kv.ref(), kv.seq_offsets_dev.data_ptr(), _ptr(kv.k), _ptr(kv.v), _ptr(k_new),
                             _ptr(v_new), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ts_decode_step_kernels(kv: KVCache, k: int, n_sink: int, n_local: int) -> int:
    """Kernels one ts_decode_step call on this cache launches."""
    n = _lib.ts_decode_step_kernels(kv.ref(), k, n_sink, n_local)
    if n < 0:
        raise TsError(TS_ERR_INVALID_ARG, ts_last_error())
    return int(n)


def ts_get_device_status(ws, stream=None):
    """Returns (status, site); status is TS_OK, TS_ERR_DEVICE_TIMEOUT (a bounded
    device wait gave up) or TS_ERR_INVALID_ARG (ts_append_kv found the cache
    full)."""
    site = ctypes.c_uint32(0)
    s = _lib.ts_get_device_status(_ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(site),
                                  _stream(stream))
    if s not in (TS_OK, TS_ERR_DEVICE_TIMEOUT, TS_ERR_INVALID_ARG):
        _check(s)
    return int(s), int(site.value)


def ts_selftest_expire_wait(ws, spin_limit: int, stream=None):
    _check(_lib.ts_selftest_expire_wait(_ptr(ws), ws.numel() * ws.element_size(), spin_limit,
                                        _stream(stream)))


# ---- token-axis split of one sequence (the joins; see split.py) ----

def ts_score_normalisers(kv: KVCache, q, reuse, L_out, ws, stream=None):
    _check(_lib.ts_score_normalisers(kv.ref(), _ptr(q), _ptr(reuse), _ptr(L_out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def ts_score_vote_normalised(kv: KVCache, reuse, L_in, votes, ws, stream=None):
    _check(_lib.ts_score_vote_normalised(kv.ref(), _ptr(reuse), _ptr(L_in), _ptr(votes), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)))


def ts_merge_normalisers(L_parts, parts: int, L_out, stream=None):
    _check(_lib.ts_merge_normalisers(_ptr(L_parts), int(parts), L_out.numel(), _ptr(L_out), _stream(stream)))


def ts_select_candidates(kv: KVCache, votes, k: int, n_sink: int, n_local: int, shard_offset: int, n_global: int,
                         ids, count, keys_out, ws, stream=None):
    _check(_lib.ts_select_candidates(kv.ref(), _ptr(votes), k, n_sink, n_local, int(shard_offset), int(n_global),
                                     _ptr(ids), _ptr(count), _ptr(keys_out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def ts_select_merge(kv: KVCache, keys_all, parts: int, rank: int, k: int, n_sink: int, n_local: int,
                    shard_offset: int, n_global: int, ids, count, stream=None):
    _check(_lib.ts_select_merge(kv.ref(), _ptr(keys_all), int(parts), int(rank), k, n_sink, n_local,
                                int(shard_offset), int(n_global), _ptr(ids), _ptr(count), _stream(stream)))


def ts_sparse_attn_lse(kv: KVCache, q, ids, count, out, lse_out, ws, stream=None):
    _check(_lib.ts_sparse_attn_lse(kv.ref(), _ptr(q), _ptr(ids), _ptr(count), ids.shape[-1], _ptr(out),
                                   _ptr(lse_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ts_merge_attention(out_parts, lse_parts, parts: int, out, stream=None):
    rows, d = lse_parts.shape[-1], out.shape[-1]
    _check(_lib.ts_merge_attention(_ptr(out_parts), _ptr(lse_parts), int(parts), rows, d, _ptr(out),
                                   _stream(stream)))


def ts_quest_rows(kv: KVCache, page_size: int) -> int:
    """Rows of the page metadata and scores: floor(n_total / P) + batch."""
    n = _lib.ts_quest_rows(kv.ref(), int(page_size))
    if n < 0:
        raise TsError(TS_ERR_INVALID_ARG, ts_last_error())
    return int(n)


def ts_quest_metadata(kv: KVCache, page_size: int, kmin, kmax, stream=None):
    _check(_lib.ts_quest_metadata(kv.ref(), int(page_size), _ptr(kmin), _ptr(kmax), _stream(stream)))


def ts_quest_metadata_update(kv: KVCache, page_size: int, last_tokens: int, kmin, kmax, stream=None):
    _check(_lib.ts_quest_metadata_update(kv.ref(), int(page_size), int(last_tokens), _ptr(kmin), _ptr(kmax),
                                         _stream(stream)))


def ts_quest_score(kv: KVCache, q, page_size: int, kmin, kmax, scores, stream=None):
    _check(_lib.ts_quest_score(kv.ref(), _ptr(q), int(page_size), _ptr(kmin), _ptr(kmax), _ptr(scores),
                               _stream(stream)))


def ts_quest_select(kv: KVCache, scores, page_size: int, k: int, n_sink: int, n_local: int, ids, count,
                    stream=None):
    _check(_lib.ts_quest_select(kv.ref(), _ptr(scores), int(page_size), int(k), int(n_sink), int(n_local),
                                _ptr(ids), _ptr(count), _stream(stream)))


def ts_status_string(status: int) -> str:
    return _status_name(status)


def ts_last_error() -> str:
    return _lib.ts_last_error().decode()


# ---------------------------------------------------------------------------
# Buffers for one decode layer-step (allocation helper; no compute)
# ---------------------------------------------------------------------------

class StepBuffers:
    """Device buffers of one layer-step: workspace, votes, ids, count, out,
    reuse flags and the selection-cache state (q_prev)."""

    def __init__(self, kv: KVCache, k: int, n_sink: int, n_local: int):
        dev = kv.k.device
        self.k, self.n_sink, self.n_local = k, n_sink, n_local
        self.capacity = k + n_sink + n_local
        nbytes = ts_workspace_bytes(kv, k, n_sink, n_local)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        ts_workspace_init(self.ws)
        self.votes = torch.zeros(max(kv.n_total, kv.capacity, 1), dtype=torch.float32, device=dev)
        self.ids = torch.full((kv.batch, self.capacity), -1, dtype=torch.int32, device=dev)
        self.count = torch.zeros(kv.batch, dtype=torch.int32, device=dev)
        self.out = torch.zeros((kv.batch, kv.h_q, kv.head_dim), dtype=torch.float32, device=dev)
        self.reuse = torch.zeros(kv.batch, dtype=torch.int32, device=dev)
        self.cos = torch.zeros(kv.batch, dtype=torch.float64, device=dev)
        self.q_prev = torch.zeros((kv.batch, kv.h_q, kv.head_dim), dtype=torch.bfloat16, device=dev)


def decode_step(kv: KVCache, q, buf: StepBuffers, *, theta=None, first_step=True, stream=None, fused=False):
    """One layer-step through the four entry points, in stream order:
    ts_selcache (when theta is given) -> ts_score -> ts_select -> ts_sparse_attn;
    fused=True makes the same step one ts_decode_step call (a theta that the
    cosine never reaches when theta is None)."""
    if fused:
        ts_decode_step(kv, q, buf.q_prev, buf.reuse, first_step, 2.0 if theta is None else theta, buf.k,
                       buf.n_sink, buf.n_local, buf.votes, buf.ids, buf.count, buf.out, buf.ws, buf.cos, stream)
        return buf.out
    reuse = None
    if theta is not None:
        ts_selcache(q, buf.q_prev, buf.reuse, first_step, theta, buf.cos, stream)
        reuse = buf.reuse
    ts_score(kv, q, reuse, buf.votes, buf.ws, stream)
    ts_select(kv, buf.votes, buf.k, buf.n_sink, buf.n_local, reuse, buf.ids, buf.count, buf.ws, stream)
    ts_sparse_attn(kv, q, buf.ids, buf.count, buf.out, buf.ws, stream)
    return buf.out


class QuestBuffers:
    """Device buffers of the page-level comparator for one cache and page
    size: the page metadata (kmin, kmax) and the page scores."""

    def __init__(self, kv: KVCache, page_size: int):
        rows = ts_quest_rows(kv, page_size)
        dev = kv.k.device
        self.page_size = int(page_size)
        self.rows = rows
        self.kmin = torch.empty((rows, kv.h_kv, kv.head_dim), dtype=torch.bfloat16, device=dev)
        self.kmax = torch.empty((rows, kv.h_kv, kv.head_dim), dtype=torch.bfloat16, device=dev)
        self.scores = torch.empty(rows, dtype=torch.float32, device=dev)


def quest_step(kv: KVCache, q, qbuf: QuestBuffers, buf: StepBuffers, stream=None):
    """Page scores -> page selection -> sparse attention, in stream order
    (the metadata is computed beforehand with ts_quest_metadata); the ids,
    count and output land in buf like decode_step's."""
    ts_quest_score(kv, q, qbuf.page_size, qbuf.kmin, qbuf.kmax, qbuf.scores, stream)
    ts_quest_select(kv, qbuf.scores, qbuf.page_size, buf.k, buf.n_sink, buf.n_local, buf.ids, buf.count, stream)
    ts_sparse_attn(kv, q, buf.ids, buf.count, buf.out, buf.ws, stream)
    return buf.out
