"""TokenSelect decode-step oracle (float64, CPU) -- Python wrapper.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never uses it, and it imports nothing from the
``query_aware_kv_ts_b200`` package.

The arithmetic lives in ``ts_oracle.c`` (plain float64 loops, compiled with
``-O2 -ffp-contract=off``, no fast-math).  This wrapper only marshals numpy
arrays and loops over the sequences of a batch.  Inputs are bf16 bit patterns
held in ``numpy.uint16`` arrays.

Sources: the TokenSelect GitHub README ("Key Takeaways": per-head Q.K
criticality, per-head soft voting, Selection Cache) and the GrooveSquid summary
of the TokenSelect paper; for the page-level comparator (``quest_*``), the
Bohrium page for Quest (arXiv 2406.10774), Abstract and "Method Overview".
Readings of the open points are listed at each function in ``ts_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ts_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_ts_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ts_oracle.c into _ts_oracle.so (gcc) when it is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _declare(lib):
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.oracle_cosine.argtypes = [P, P, i64]
    lib.oracle_cosine.restype = f64
    lib.oracle_selcache.argtypes = [P, P, i64, ctypes.c_int, f64, P]
    lib.oracle_selcache.restype = ctypes.c_int
    lib.oracle_head_logits.argtypes = [P, i64, i32, i32, i64, i64, P, i32, i32, f64, P]
    lib.oracle_head_logits.restype = None
    lib.oracle_softmax_row.argtypes = [P, i64, P]
    lib.oracle_softmax_row.restype = f64
    lib.oracle_votes.argtypes = [P, i64, i32, i32, i64, i64, P, i32, f64, P, P]
    lib.oracle_votes.restype = None
    lib.oracle_windows.argtypes = [i64, i64, i64, P, P]
    lib.oracle_windows.restype = None
    lib.oracle_select.argtypes = [P, i64, i64, i64, i64, P]
    lib.oracle_select.restype = i64
    lib.oracle_reuse_ids.argtypes = [P, i64, i64, i64, i64, i64, i64, P]
    lib.oracle_reuse_ids.restype = i64
    lib.oracle_sparse_attn.argtypes = [P, P, i32, i32, i64, i64, P, i32, f64, P, i64, P]
    lib.oracle_sparse_attn.restype = None
    lib.oracle_dense_attn.argtypes = [P, P, i64, i32, i32, i64, i64, P, i32, f64, P]
    lib.oracle_dense_attn.restype = None
    lib.oracle_quest_pages.argtypes = [i64, i64]
    lib.oracle_quest_pages.restype = i64
    lib.oracle_quest_meta.argtypes = [P, i64, i32, i32, i64, i64, i64, P, P]
    lib.oracle_quest_meta.restype = None
    lib.oracle_quest_scores.argtypes = [P, P, i64, i32, i32, P, i32, f64, P]
    lib.oracle_quest_scores.restype = None
    lib.oracle_quest_select.argtypes = [P, i64, i64, i64, i64, i64, P]
    lib.oracle_quest_select.restype = i64
    return lib


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


class using_library:
    """Context manager: run the wrapper against another build of ts_oracle.c
    (the pin-strength tests compile deliberately broken copies of the oracle
    and check that the pins reject them)."""

    def __init__(self, path: str):
        self._path = path
        self._saved = None

    def __enter__(self):
        global _lib
        lib()
        with _lock:
            self._saved = _lib
            _lib = _declare(ctypes.CDLL(self._path))
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved
        return False


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns, got %s" % a.dtype)
    return a


def _kv_view(k: np.ndarray):
    """k: uint16 [tokens, h_kv, d] with arbitrary (element) strides."""
    k = _u16(k)
    if k.ndim != 3 or k.strides[2] != 2:
        raise ValueError("K/V must be [tokens, h_kv, d] with contiguous channels")
    return k, k.strides[0] // 2, k.strides[1] // 2


def default_scale(d: int) -> float:
    return 1.0 / np.sqrt(float(d))


# ---------------------------------------------------------------------------
# Single-sequence definitions
# ---------------------------------------------------------------------------

def cosine(a, b) -> float:
    a = np.ascontiguousarray(_u16(a)).reshape(-1)
    b = np.ascontiguousarray(_u16(b)).reshape(-1)
    assert a.size == b.size
    return float(lib().oracle_cosine(_ptr(a), _ptr(b), a.size))


def selcache(q, q_prev: np.ndarray, first_step: bool, theta: float):
    """Selection-cache decision for one sequence; updates q_prev in place.

    Returns (reuse: bool, cosine: float)."""
    q = np.ascontiguousarray(_u16(q)).reshape(-1)
    assert q_prev.flags.c_contiguous and q_prev.dtype == np.uint16 and q_prev.size == q.size
    c = ctypes.c_double(0.0)
    r = lib().oracle_selcache(_ptr(q), _ptr(q_prev), q.size, int(bool(first_step)),
                              float(theta), ctypes.byref(c))
    return bool(r), float(c.value)


def head_logits(k, q, h: int, scale: float | None = None) -> np.ndarray:
    k, st, sh = _kv_view(k)
    q = np.ascontiguousarray(_u16(q))
    n, h_kv, d = k.shape
    h_q = q.shape[0]
    s = np.empty(n, np.float64)
    lib().oracle_head_logits(_ptr(k), n, h_kv, d, st, sh, _ptr(q), h_q, h,
                             default_scale(d) if scale is None else float(scale), _ptr(s))
    return s


def softmax_row(s) -> tuple[np.ndarray, float]:
    s = np.ascontiguousarray(s, dtype=np.float64)
    p = np.empty_like(s)
    L = lib().oracle_softmax_row(_ptr(s), s.size, _ptr(p))
    return p, float(L)


def votes(k, q, scale: float | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Soft vote v[n] and per-head log-normalisers L[h_q] of one sequence."""
    k, st, sh = _kv_view(k)
    q = np.ascontiguousarray(_u16(q))
    n, h_kv, d = k.shape
    h_q = q.shape[0]
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    v = np.empty(n, np.float64)
    L = np.empty(h_q, np.float64)
    lib().oracle_votes(_ptr(k), n, h_kv, d, st, sh, _ptr(q), h_q,
                       default_scale(d) if scale is None else float(scale), _ptr(v), _ptr(L))
    return v, L


def windows(n: int, n_sink: int, n_local: int) -> tuple[int, int]:
    a, b = ctypes.c_int64(), ctypes.c_int64()
    lib().oracle_windows(n, n_sink, n_local, ctypes.byref(a), ctypes.byref(b))
    return int(a.value), int(b.value)


def select(v, k: int, n_sink: int, n_local: int) -> tuple[np.ndarray, int]:
    """Ascending selected ids (padded with -1 to k+s+l) and their count."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    ids = np.empty(k + n_sink + n_local, np.int32)
    m = lib().oracle_select(_ptr(v), v.size, k, n_sink, n_local, _ptr(ids))
    return ids, int(m)


def reuse_ids(prev_ids, prev_count: int, n_old: int, n_new: int, k: int, n_sink: int,
              n_local: int) -> tuple[np.ndarray, int]:
    """The ids of a sequence that reuses its selection after its cache grew from
    n_old to n_new tokens: the previous top-k part with the current sink and
    local windows (reading R19; the previous row itself when n_new == n_old).
    Returns (ids int32 [k + n_sink + n_local] with -1 padding, count)."""
    prev = np.ascontiguousarray(prev_ids, dtype=np.int32)
    out = np.empty(k + n_sink + n_local, np.int32)
    m = lib().oracle_reuse_ids(_ptr(prev), int(prev_count), int(n_old), int(n_new), k, n_sink, n_local, _ptr(out))
    return out, int(m)


def sparse_attn(k, v, q, ids, m: int | None = None, scale: float | None = None) -> np.ndarray:
    k, st, sh = _kv_view(k)
    v, vst, vsh = _kv_view(v)
    if (vst, vsh) != (st, sh) or v.shape != k.shape:
        raise ValueError("K and V must share shape and strides")
    q = np.ascontiguousarray(_u16(q))
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    if m is None:
        m = ids.size
    n, h_kv, d = k.shape
    if m and (ids[:m].min() < 0 or ids[:m].max() >= n):
        raise ValueError("ids out of range")
    h_q = q.shape[0]
    out = np.empty((h_q, d), np.float64)
    lib().oracle_sparse_attn(_ptr(k), _ptr(v), h_kv, d, st, sh, _ptr(q), h_q,
                             default_scale(d) if scale is None else float(scale),
                             _ptr(ids), int(m), _ptr(out))
    return out


def dense_attn(k, v, q, scale: float | None = None) -> np.ndarray:
    k, st, sh = _kv_view(k)
    v, vst, vsh = _kv_view(v)
    if (vst, vsh) != (st, sh) or v.shape != k.shape:
        raise ValueError("K and V must share shape and strides")
    q = np.ascontiguousarray(_u16(q))
    n, h_kv, d = k.shape
    h_q = q.shape[0]
    out = np.empty((h_q, d), np.float64)
    lib().oracle_dense_attn(_ptr(k), _ptr(v), n, h_kv, d, st, sh, _ptr(q), h_q,
                            default_scale(d) if scale is None else float(scale), _ptr(out))
    return out


# ---------------------------------------------------------------------------
# One decode layer-step over a (ragged) batch
# ---------------------------------------------------------------------------

class StepResult:
    __slots__ = ("reuse", "cos", "votes", "L", "ids", "count", "out")

    def __init__(self, B):
        self.reuse = np.zeros(B, bool)
        self.cos = np.zeros(B, np.float64)
        self.votes = []
        self.L = []
        self.ids = []
        self.count = np.zeros(B, np.int64)
        self.out = []


def decode_step(k, v, seq_offsets, q, k_top: int, n_sink: int, n_local: int,
                *, q_prev=None, prev_ids=None, first_step=True, theta=None,
                reuse_override=None, scale=None) -> StepResult:
    """Selection cache -> soft vote -> selection -> sparse attention, per sequence.

    k, v: uint16 [sum_n, h_kv, d]; seq_offsets: int64 [B+1]; q: uint16 [B, h_q, d].
    q_prev: uint16 [B, h_q, d] state, updated in place when theta is not None.
    prev_ids: list of the previous step's id arrays (used when a sequence reuses).
    reuse_override: optional bool[B] that replaces the cosine decision (used when
    the cosine sits within rounding distance of theta).
    """
    seq_offsets = np.asarray(seq_offsets, dtype=np.int64)
    B = seq_offsets.size - 1
    res = StepResult(B)
    for b in range(B):
        lo, hi = int(seq_offsets[b]), int(seq_offsets[b + 1])
        kb, vb, qb = k[lo:hi], v[lo:hi], q[b]
        reuse = False
        if theta is not None:
            reuse, c = selcache(qb, q_prev[b], first_step, theta)
            res.cos[b] = c
        if reuse_override is not None:
            reuse = bool(reuse_override[b])
        res.reuse[b] = reuse
        if reuse:
            if prev_ids is None:
                raise ValueError("reuse needs the previous ids")
            ids = np.asarray(prev_ids[b], dtype=np.int32)
            m = int((ids >= 0).sum())
            res.votes.append(None)
            res.L.append(None)
        else:
            vb_votes, L = votes(kb, qb, scale)
            ids, m = select(vb_votes, k_top, n_sink, n_local)
            res.votes.append(vb_votes)
            res.L.append(L)
        res.ids.append(ids)
        res.count[b] = m
        res.out.append(sparse_attn(kb, vb, qb, ids, m, scale))
    return res


# ---------------------------------------------------------------------------
# A decode loop over one growing sequence
# ---------------------------------------------------------------------------

def decode_loop(k, v, n0: int, qs, k_top: int, n_sink: int, n_local: int, theta: float,
                scale=None, reuse_override=None) -> list[dict]:
    """One layer of one sequence over T decode steps with KV append (reading
    R19): step t attends over the first n_t = n0 + t tokens of k, v (the token
    appended before the step included).  The selection cache compares q_t with
    q_{t-1} (never at t = 0); on reuse the ids are reuse_ids() of the previous
    step's row, otherwise the full vote and selection over the n_t tokens.

    k, v: uint16 [>= n0 + T - 1, h_kv, d]; qs: uint16 [T, h_q, d].
    reuse_override: optional bool [T] replacing the cosine decision.
    Returns one dict per step: reuse, cos, n, ids, count, out (and votes when
    the selection was recomputed)."""
    k, v, qs = _u16(k), _u16(v), _u16(qs)
    T = qs.shape[0]
    q_prev = np.zeros_like(qs[0])
    steps = []
    prev = None
    for t in range(T):
        n_t = n0 + t
        reuse, c = selcache(qs[t], q_prev, t == 0, theta)
        if reuse_override is not None:
            reuse = bool(reuse_override[t])
        kb, vb = k[:n_t], v[:n_t]
        rec = {"reuse": reuse, "cos": c, "n": n_t}
        if reuse:
            ids, m = reuse_ids(prev["ids"], prev["count"], prev["n"], n_t, k_top, n_sink, n_local)
        else:
            vt, _ = votes(kb, qs[t], scale)
            ids, m = select(vt, k_top, n_sink, n_local)
            rec["votes"] = vt
        rec["ids"], rec["count"] = ids, m
        rec["out"] = sparse_attn(kb, vb, qs[t], ids, m, scale)
        steps.append(rec)
        prev = rec
    return steps


# ---------------------------------------------------------------------------
# Page-level comparator (Quest's min/max page bounds)
# ---------------------------------------------------------------------------

def quest_pages(n: int, page_size: int) -> int:
    """Pages of a sequence of n tokens: ceil(n / page_size)."""
    return int(lib().oracle_quest_pages(int(n), int(page_size)))


def quest_meta(k, page_size: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-page element-wise (min, max) of one sequence's keys, bf16 bits
    [pages, h_kv, d] each."""
    k, st, sh = _kv_view(k)
    n, h_kv, d = k.shape
    pages = quest_pages(n, page_size)
    kmin = np.empty((pages, h_kv, d), np.uint16)
    kmax = np.empty((pages, h_kv, d), np.uint16)
    lib().oracle_quest_meta(_ptr(k), n, h_kv, d, st, sh, int(page_size), _ptr(kmin), _ptr(kmax))
    return kmin, kmax


def quest_scores(kmin, kmax, q, scale: float | None = None) -> np.ndarray:
    """Page scores (float64 [pages]): the per-head upper bounds of the scaled
    logit over each page's min/max box, summed over the query heads."""
    kmin = np.ascontiguousarray(_u16(kmin))
    kmax = np.ascontiguousarray(_u16(kmax))
    q = np.ascontiguousarray(_u16(q))
    pages, h_kv, d = kmin.shape
    h_q = q.shape[0]
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    out = np.empty(pages, np.float64)
    lib().oracle_quest_scores(_ptr(kmin), _ptr(kmax), pages, h_kv, d, _ptr(q), h_q,
                              default_scale(d) if scale is None else float(scale), _ptr(out))
    return out


def quest_select(scores, n: int, page_size: int, k: int, n_sink: int, n_local: int) -> tuple[np.ndarray, int]:
    """Ascending ids (padded with -1 to k+s+l) and their count: the sink and
    local windows plus the candidate tokens of the top floor(k / page_size)
    candidate pages."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    assert scores.size == quest_pages(n, page_size)
    ids = np.empty(k + n_sink + n_local, np.int32)
    m = lib().oracle_quest_select(_ptr(scores), int(n), int(page_size), int(k), int(n_sink), int(n_local),
                                  _ptr(ids))
    return ids, int(m)


def quest_step(k, v, q, page_size: int, k_top: int, n_sink: int, n_local: int,
               scale: float | None = None):
    """One sequence's page-level step: metadata, page scores, selection and
    attention over the selected tokens.  Returns (scores, ids, count, out)."""
    kmin, kmax = quest_meta(k, page_size)
    sc = quest_scores(kmin, kmax, q, scale)
    ids, m = quest_select(sc, k.shape[0], page_size, k_top, n_sink, n_local)
    out = sparse_attn(k, v, q, ids, m, scale)
    return sc, ids, m, out
