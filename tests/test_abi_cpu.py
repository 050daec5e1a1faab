"""The C-ABI library loads and exports every function include/ts.h declares.

Runs without a GPU: only symbol lookup and argument checks that fail on the
host before any CUDA call are exercised here (no compute)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ts.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"TS_API\s+[\w\s\*]+?\b(ts_\w+)\s*\(", src)))


def load_build_module():
    import importlib.util
    path = os.path.join(ROOT, "query_aware_kv_ts_b200", "csrc", "build.py")
    spec = importlib.util.spec_from_file_location("ts_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(load_build_module().build())


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("ts_selcache", "ts_score", "ts_select", "ts_sparse_attn", "ts_workspace_bytes",
                 "ts_get_device_status", "ts_status_string"):
        assert want in names, names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_only_declared_symbols_are_exported(lib):
    out = os.popen("nm -D --defined-only %s" % lib._name).read()
    exported = sorted(set(re.findall(r"\b[TW] (ts_\w+)", out)))
    assert exported == _declared(), (exported, _declared())


def test_status_strings(lib):
    lib.ts_status_string.restype = ctypes.c_char_p
    for code, name in enumerate(["TS_OK", "TS_ERR_INVALID_ARG", "TS_ERR_UNSUPPORTED", "TS_ERR_WORKSPACE",
                                 "TS_ERR_CUDA", "TS_ERR_DEVICE_TIMEOUT"]):
        assert lib.ts_status_string(code).decode() == name


def test_host_side_argument_errors(lib):
    """Invalid arguments are rejected on the host before anything is launched."""
    lib.ts_last_error.restype = ctypes.c_char_p
    lib.ts_score.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_size_t, ctypes.c_void_p]
    assert lib.ts_score(None, None, None, None, None, 0, None) == 1          # votes NULL
    assert lib.ts_last_error() != b""
    lib.ts_score_logits.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_size_t, ctypes.c_void_p]
    assert lib.ts_score_logits(None, None, None, None, 0, None) == 1       # kv NULL
    assert b"kv" in lib.ts_last_error()
    lib.ts_selcache.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int32] * 4 + [ctypes.c_double, ctypes.c_void_p]
    assert lib.ts_selcache(None, None, None, None, 0, 1, 4, 64, 0.9, None) == 1
    lib.ts_workspace_init.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert lib.ts_workspace_init(None, 0, None) == 3
    lib.ts_selftest_expire_wait.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_void_p]
    assert lib.ts_selftest_expire_wait(None, 0, 10, None) == 3


class _KV(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("seq_offsets_dev", ctypes.c_void_p),
                ("seq_offsets_host", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("stride_tok", ctypes.c_int64), ("stride_head", ctypes.c_int64), ("scale", ctypes.c_float),
                ("capacity", ctypes.c_int64), ("page_size", ctypes.c_int32),
                ("page_table_stride", ctypes.c_int32), ("pool_pages", ctypes.c_int64),
                ("page_table_dev", ctypes.c_void_p)]


def test_decode_step_checks_everything_before_launching(lib):
    """ts_decode_step validates its whole argument list on the host: nothing
    is launched (no GPU is touched here) when any argument is wrong."""
    lib.ts_last_error.restype = ctypes.c_char_p
    P, I32, F64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double, ctypes.c_size_t
    lib.ts_decode_step.argtypes = [ctypes.POINTER(_KV), P, P, P, P, I32, F64, I32, I32, I32, P, P, P, P, P, SZ, P]

    def call(kv, k=16, s=4, l=8):
        return lib.ts_decode_step(kv, None, None, None, None, 1, 0.9, k, s, l, None, None, None, None, None, 0,
                                  None)

    assert call(None, k=-1) == 1 and b"non-negative" in lib.ts_last_error()
    assert call(None, k=0, s=0, l=0) == 1                     # empty selection capacity
    assert call(None) == 1 and b"kv" in lib.ts_last_error()
    off = (ctypes.c_int64 * 2)(0, 64)
    kv = _KV(1, 6, 4, 64, ctypes.addressof(off), ctypes.addressof(off), 16, 16, 256, 64, 0.0)
    assert call(ctypes.byref(kv)) == 1 and b"multiple" in lib.ts_last_error()   # h_q % h_kv
    kv = _KV(1, 8, 4, 96, ctypes.addressof(off), ctypes.addressof(off), 16, 16, 384, 96, 0.0)
    assert call(ctypes.byref(kv)) == 2                         # head_dim 96: unsupported
    kv = _KV(1, 8, 4, 64, ctypes.addressof(off), ctypes.addressof(off), 8, 16, 256, 64, 0.0)
    assert call(ctypes.byref(kv)) == 1 and b"16-byte" in lib.ts_last_error()    # misaligned K


def test_decode_step_kernels_rejects_bad_arguments(lib):
    """ts_decode_step_kernels answers -1 (with an error message) for invalid
    selection sizes or a missing cache, before any device query."""
    lib.ts_last_error.restype = ctypes.c_char_p
    lib.ts_decode_step_kernels.restype = ctypes.c_int32
    lib.ts_decode_step_kernels.argtypes = [ctypes.POINTER(_KV), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    assert lib.ts_decode_step_kernels(None, -1, 4, 8) == -1 and b"non-negative" in lib.ts_last_error()
    assert lib.ts_decode_step_kernels(None, 0, 0, 0) == -1
    assert lib.ts_decode_step_kernels(None, 16, 4, 8) == -1 and b"kv" in lib.ts_last_error()


def test_binding_refuses_host_tensors():
    """No CPU path: the binding refuses host tensors before calling the library."""
    import torch

    import query_aware_kv_ts_b200 as ts
    k = torch.zeros((64, 4, 64), dtype=torch.bfloat16)
    kv = ts.KVCache(k, k.clone(), [0, 64], 8)
    q = torch.zeros((1, 8, 64), dtype=torch.bfloat16)
    votes = torch.zeros(64)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="GPU only"):
        ts.ts_score(kv, q, None, votes, ws)
    with pytest.raises(ValueError, match="GPU only"):
        ts.ts_selcache(q, q.clone(), torch.zeros(1, dtype=torch.int32), True, 0.9)


def test_growing_cache_arguments_are_checked_on_the_host(lib):
    """A cache with a capacity: one sequence only, capacity >= the current
    length, and ts_append_kv refuses a cache without one; all decided on the
    host before any device query."""
    lib.ts_last_error.restype = ctypes.c_char_p
    lib.ts_decode_step_kernels.restype = ctypes.c_int32
    lib.ts_decode_step_kernels.argtypes = [ctypes.POINTER(_KV), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    off1 = (ctypes.c_int64 * 2)(0, 64)
    off2 = (ctypes.c_int64 * 3)(0, 64, 128)
    kv = _KV(1, 8, 4, 64, ctypes.addressof(off1), ctypes.addressof(off1), 16, 16, 256, 64, 0.0, -1)
    assert lib.ts_decode_step_kernels(ctypes.byref(kv), 16, 4, 8) == -1 and b">= 0" in lib.ts_last_error()
    kv = _KV(2, 8, 4, 64, ctypes.addressof(off2), ctypes.addressof(off2), 16, 16, 256, 64, 0.0, 4096)
    assert lib.ts_decode_step_kernels(ctypes.byref(kv), 16, 4, 8) == -1 and b"one sequence" in lib.ts_last_error()
    kv = _KV(1, 8, 4, 64, ctypes.addressof(off1), ctypes.addressof(off1), 16, 16, 256, 64, 0.0, 32)
    assert lib.ts_decode_step_kernels(ctypes.byref(kv), 16, 4, 8) == -1 and b"below" in lib.ts_last_error()
    P = ctypes.c_void_p
    lib.ts_append_kv.argtypes = [ctypes.POINTER(_KV), P, P, P, P, P, P, ctypes.c_size_t, P]
    kv = _KV(1, 8, 4, 64, ctypes.addressof(off1), ctypes.addressof(off1), 16, 16, 256, 64, 0.0, 0)
    assert lib.ts_append_kv(ctypes.byref(kv), None, None, None, None, None, None, 0, None) == 1


def test_paged_cache_arguments_are_checked_on_the_host(lib):
    """A paged cache: page size a power of two in [8, 4096], no capacity, a
    block table with a row per sequence wide enough for the longest one, and
    a pool below 2^31 rows; all decided on the host before any device query."""
    lib.ts_last_error.restype = ctypes.c_char_p
    lib.ts_decode_step_kernels.restype = ctypes.c_int32
    lib.ts_decode_step_kernels.argtypes = [ctypes.POINTER(_KV), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    off = (ctypes.c_int64 * 3)(0, 100, 130)
    table = (ctypes.c_int32 * 64)()

    def kv(page, stride, pool, capacity=0, tab=ctypes.addressof(table)):
        return _KV(2, 8, 4, 64, ctypes.addressof(off), ctypes.addressof(off), 16, 16, 256, 64, 0.0, capacity,
                   page, stride, pool, tab)

    for page in (4, 24, 8192):
        assert lib.ts_decode_step_kernels(ctypes.byref(kv(page, 32, 64)), 16, 4, 8) == -1
        assert b"page_size" in lib.ts_last_error()
    assert lib.ts_decode_step_kernels(ctypes.byref(kv(16, 32, 64, capacity=200)), 16, 4, 8) == -1
    assert b"capacity" in lib.ts_last_error()
    assert lib.ts_decode_step_kernels(ctypes.byref(kv(16, 32, 64, tab=None)), 16, 4, 8) == -1
    assert b"page_table_dev" in lib.ts_last_error()
    # the longest sequence (100 tokens) needs 7 pages of 16
    assert lib.ts_decode_step_kernels(ctypes.byref(kv(16, 6, 64)), 16, 4, 8) == -1
    assert b"page_table_stride" in lib.ts_last_error()
    assert lib.ts_decode_step_kernels(ctypes.byref(kv(4096, 1, 1 << 19)), 16, 4, 8) == -1
    assert b"2^31" in lib.ts_last_error()


def test_split_and_comparator_arguments_are_checked_on_the_host(lib):
    """The page-level comparator's and the token split's entry points reject
    bad arguments on the host, before any device query or launch."""
    lib.ts_last_error.restype = ctypes.c_char_p
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    off1 = (ctypes.c_int64 * 2)(0, 500)
    off2 = (ctypes.c_int64 * 3)(0, 500, 900)
    one = _KV(1, 8, 4, 64, ctypes.addressof(off1), ctypes.addressof(off1), 16, 16, 256, 64, 0.0, 0)
    two = _KV(2, 8, 4, 64, ctypes.addressof(off2), ctypes.addressof(off2), 16, 16, 256, 64, 0.0, 0)
    lib.ts_quest_rows.restype = I64
    lib.ts_quest_rows.argtypes = [ctypes.POINTER(_KV), I32]
    for page in (0, 3, 8192):
        assert lib.ts_quest_rows(ctypes.byref(one), page) == -1 and b"page_size" in lib.ts_last_error()
    assert lib.ts_quest_rows(None, 16) == -1
    lib.ts_quest_metadata_update.argtypes = [ctypes.POINTER(_KV), I32, I64, P, P, P]
    for last in (0, -5):
        assert lib.ts_quest_metadata_update(ctypes.byref(one), 16, last, None, None, None) == 1
        assert b"last_tokens" in lib.ts_last_error()
    assert lib.ts_quest_metadata_update(ctypes.byref(one), 3, 1, None, None, None) == 1
    assert b"page_size" in lib.ts_last_error()
    lib.ts_merge_normalisers.argtypes = [P, I32, I64, P, P]
    assert lib.ts_merge_normalisers(None, 2, 8, None, None) == 1
    lib.ts_merge_attention.argtypes = [P, P, I32, I64, I32, P, P]
    assert lib.ts_merge_attention(None, None, 2, 8, 64, None, None) == 1
    lib.ts_score_normalisers.argtypes = [ctypes.POINTER(_KV), P, P, P, P, SZ, P]
    assert lib.ts_score_normalisers(ctypes.byref(one), None, None, None, None, 0, None) == 1
    assert b"L_out" in lib.ts_last_error()
    lib.ts_select_candidates.argtypes = [ctypes.POINTER(_KV), P, I32, I32, I32, I64, I64, P, P, P, P, SZ, P]
    # k < 1; a batch of two sequences; a shard reaching past the sequence
    assert lib.ts_select_candidates(ctypes.byref(one), None, 0, 4, 8, 0, 500, None, None, None, None, 0, None) == 1
    assert lib.ts_select_candidates(ctypes.byref(two), None, 16, 4, 8, 0, 900, None, None, None, None, 0, None) == 1
    assert b"batch 1" in lib.ts_last_error()
    assert lib.ts_select_candidates(ctypes.byref(one), None, 16, 4, 8, 600, 1000, None, None, None, None, 0,
                                    None) == 1
    assert b"must lie in the sequence" in lib.ts_last_error()
    lib.ts_select_merge.argtypes = [ctypes.POINTER(_KV), P, I32, I32, I32, I32, I32, I64, I64, P, P, P]
    # rank outside [0, parts)
    assert lib.ts_select_merge(ctypes.byref(one), None, 2, 2, 16, 4, 8, 0, 1000, None, None, None) == 1
    lib.ts_sparse_attn_lse.argtypes = [ctypes.POINTER(_KV), P, P, P, I32, P, P, P, SZ, P]
    assert lib.ts_sparse_attn_lse(ctypes.byref(one), None, None, None, 0, None, None, None, 0, None) == 1
