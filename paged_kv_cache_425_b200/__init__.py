"""Python binding of libpa.so (paged KV-cache decode for B200, sm_100a).

Argument marshalling only: each function checks that the tensors it is given
have the documented shape, type and device, then calls the C entry point of
the same name (include/pa_api.h, include/pa_alloc.h).  Every step of the hot
path runs in the library's CUDA kernels; there is no CPU fallback, and
importing this package fails if the library has not been built
(``python paged_kv_cache_425_b200/build.py``).

PyTorch serves only as the owner of device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

F16 = 0
BF16 = 1
BLOCK_SIZE = 16
PARTITION_TOKENS = 512
STATIC_WORKSPACE_BYTES = 48 << 20  # PA_STATIC_WORKSPACE_BYTES

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_OUT_OF_RANGE = -3
PA_ERR_NO_BLOCKS = -4
PA_ERR_CUDA = -5
PA_ERR_WORKSPACE = -6
PA_ERR_TIMEOUT = -7

DEVERR_BLOCK_ID = 1
DEVERR_SLOT = 2
DEVERR_PAIR = 4
DEVERR_CONTEXT_LEN = 8
DEVERR_TIMEOUT = 16

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python paged_kv_cache_425_b200/build.py` (no CPU fallback exists)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_i32, _i64, _f32, _f64, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_size_t


def _sig(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


class SimStats(ctypes.Structure):
    _fields_ = [("steps", _i64), ("tokens_generated", _i64), ("preemptions", _i64),
                ("admitted", _i64), ("finished", _i64), ("rejected", _i64),
                ("mean_usage", _f64), ("max_usage", _f64), ("mean_running", _f64)]


class AllocStats(ctypes.Structure):
    _fields_ = [("num_blocks", _i64), ("free_blocks", _i64), ("used_blocks", _i64),
                ("shared_blocks", _i64), ("num_seqs", _i64), ("logical_tokens", _i64),
                ("logical_blocks", _i64), ("filled_slots", _i64), ("cow_copies", _i64),
                ("cached_blocks", _i64), ("prefix_query_blocks", _i64),
                ("prefix_hit_blocks", _i64), ("usage", _f64), ("waste", _f64),
                ("sharing_saving", _f64)]


pa_reshape_and_cache = _sig("pa_reshape_and_cache", ctypes.c_int, _P, _P, _P, _P, _P, _i32, _i32,
                            _i32, _i32, _i64, _i32, _P)
pa_decode = _sig("pa_decode", ctypes.c_int, _P, _P, _P, _P, _P, _P, _i32, _f32, _i32, _i32, _i32,
                 _i32, _i32, _i64, _i32, _P, _sz, _P)
pa_decode_append = _sig("pa_decode_append", ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _P, _i32,
                        _f32, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _P, _sz, _P)
pa_decode_workspace_size = _sig("pa_decode_workspace_size", _sz, _i32, _i32, _i32, _i32, _i32)
pa_decode_static_workspace = _sig("pa_decode_static_workspace", ctypes.c_int, _P, _P, _P, _P, _P,
                                  _P, _i32, _f32, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _P)
pa_prefill = _sig("pa_prefill", ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _i32, _i32, _f32, _i32,
                  _i32, _i32, _i32, _i32, _i32, _i64, _i32, _P)
pa_prefill_select = _sig("pa_prefill_select", ctypes.c_int, _i32)
pa_copy_blocks = _sig("pa_copy_blocks", ctypes.c_int, _P, _P, _P, _i32, _i32, _i32, _i32, _i64,
                      _i32, _P)
pa_swap_blocks = _sig("pa_swap_blocks", ctypes.c_int, _P, _P, _i64, _P, _P, _i64, _P, _i32, _i32,
                      _i32, _i32, _i32, _P)
pa_get_error = _sig("pa_get_error", ctypes.c_int, _P, ctypes.POINTER(ctypes.c_uint32))
pa_selftest_wait_timeout = _sig("pa_selftest_wait_timeout", ctypes.c_int, ctypes.c_uint64, _P)
pa_status_string = _sig("pa_status_string", ctypes.c_char_p, ctypes.c_int)
pa_version = _sig("pa_version", ctypes.c_int)
pa_alloc_create = _sig("pa_alloc_create", _P, _i32, _i32)
pa_alloc_destroy = _sig("pa_alloc_destroy", None, _P)
pa_alloc_add_seq = _sig("pa_alloc_add_seq", ctypes.c_int, _P, _i64, _i32)
pa_alloc_fork = _sig("pa_alloc_fork", ctypes.c_int, _P, _i64, _i64)
pa_alloc_append_slot = _sig("pa_alloc_append_slot", ctypes.c_int, _P, _i64,
                            ctypes.POINTER(_i64), ctypes.POINTER(_i32), ctypes.POINTER(_i32))
pa_alloc_append_slots = _sig("pa_alloc_append_slots", ctypes.c_int, _P, _P, _i32, _P, _P,
                             ctypes.POINTER(_i32))
pa_alloc_free_seq = _sig("pa_alloc_free_seq", ctypes.c_int, _P, _i64)
pa_alloc_num_tokens = _sig("pa_alloc_num_tokens", _i32, _P, _i64)
pa_alloc_block_table = _sig("pa_alloc_block_table", _i32, _P, _i64, _P, _i32)
pa_alloc_build_tables = _sig("pa_alloc_build_tables", ctypes.c_int, _P, _P, _i32, _P, _i32, _P)
pa_alloc_refcount = _sig("pa_alloc_refcount", _i32, _P, _i32)
pa_alloc_enable_prefix_caching = _sig("pa_alloc_enable_prefix_caching", ctypes.c_int, _P, _i32)
pa_alloc_add_seq_tokens = _sig("pa_alloc_add_seq_tokens", ctypes.c_int, _P, _i64, _P, _i32,
                               ctypes.POINTER(_i32))
pa_alloc_get_stats = _sig("pa_alloc_get_stats", ctypes.c_int, _P, ctypes.POINTER(AllocStats))
pa_sim_continuous_batching = _sig("pa_sim_continuous_batching", ctypes.c_int, _i32, _i32, _i32,
                                  _P, _P, _i32, _i64, ctypes.POINTER(SimStats))
pa_kv_bytes_per_token = _sig("pa_kv_bytes_per_token", _i64, _i32, _i32, _i32, _i32)
pa_pool_bytes = _sig("pa_pool_bytes", _f64, _f64, _f64, _f64)
pa_pool_num_blocks = _sig("pa_pool_num_blocks", _i64, _f64, _i32, _i32, _i32, _i32, _i32)


class PagedError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {pa_status_string(status).decode()} ({status})")


def _check(rc: int, what: str):
    if rc != PA_OK:
        raise PagedError(rc, what)


# ---------------------------------------------------------------- device calls (torch tensors)
def _torch():
    import torch
    return torch


def dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtype=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _cache_shape(key_cache, value_cache):
    if key_cache.shape != value_cache.shape or key_cache.dtype != value_cache.dtype:
        raise ValueError("key_cache and value_cache must match")
    nb, hkv, bs, d = key_cache.shape
    return nb, hkv, bs, d


def reshape_and_cache(k, v, key_cache, value_cache, slot_mapping, stream=None):
    """Write k, v [T][Hkv][d] into cache slots slot_mapping [T] (int64)."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    T = int(slot_mapping.shape[0])
    for t, n in ((k, "k"), (v, "v")):
        if tuple(t.shape) != (T, hkv, d) or t.dtype != key_cache.dtype:
            raise ValueError(f"{n} must be [{T}, {hkv}, {d}] {key_cache.dtype}")
    _check(pa_reshape_and_cache(_dev(k, "k"), _dev(v, "v"), _dev(key_cache, "key_cache", ndim=4),
                                _dev(value_cache, "value_cache", ndim=4),
                                _dev(slot_mapping, "slot_mapping", torch.int64, 1), T, hkv, d, bs,
                                nb, dtype_code(key_cache), _stream(stream)), "pa_reshape_and_cache")


def decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int, max_blocks_per_seq: int,
                          block_size: int = BLOCK_SIZE) -> int:
    return int(pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                        max_blocks_per_seq))


def decode(out, q, key_cache, value_cache, block_tables, context_lens, num_kv_heads: int,
           scale: float, workspace=None, stream=None):
    """Paged decode attention: out[s][h] = softmax(scale q K^T) V over the paged context."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if hkv != num_kv_heads:
        raise ValueError("num_kv_heads does not match the cache")
    S, hq, dq = q.shape
    if dq != d or tuple(out.shape) != (S, hq, d) or out.dtype != q.dtype or q.dtype != key_cache.dtype:
        raise ValueError("q / out must be [S, Hq, d] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    maxb = int(block_tables.shape[1])
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(pa_decode(_dev(out, "out"), _dev(q, "q"), _dev(key_cache, "key_cache"),
                     _dev(value_cache, "value_cache"),
                     _dev(block_tables, "block_tables", torch.int32, 2),
                     _dev(context_lens, "context_lens", torch.int32, 1), hkv, float(scale), S, hq,
                     d, bs, maxb, nb, dtype_code(q), ws_ptr, ws_bytes, _stream(stream)),
           "pa_decode")


def decode_append(out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens,
                  num_kv_heads: int, scale: float, workspace=None, stream=None):
    """Write each sequence's new token (k_new, v_new: [S, Hkv, d]) at position
    context_lens[s] - 1 of its table, then decode, in one launch: the same
    cache bytes and outputs as reshape_and_cache followed by decode."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if hkv != num_kv_heads:
        raise ValueError("num_kv_heads does not match the cache")
    S, hq, dq = q.shape
    if dq != d or tuple(out.shape) != (S, hq, d) or out.dtype != q.dtype or q.dtype != key_cache.dtype:
        raise ValueError("q / out must be [S, Hq, d] of the cache dtype")
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if tuple(t.shape) != (S, hkv, d) or t.dtype != key_cache.dtype:
            raise ValueError(f"{name} must be [S, Hkv, d] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    maxb = int(block_tables.shape[1])
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(pa_decode_append(_dev(out, "out"), _dev(q, "q"), _dev(k_new, "k_new"),
                            _dev(v_new, "v_new"), _dev(key_cache, "key_cache"),
                            _dev(value_cache, "value_cache"),
                            _dev(block_tables, "block_tables", torch.int32, 2),
                            _dev(context_lens, "context_lens", torch.int32, 1), hkv, float(scale),
                            S, hq, d, bs, maxb, nb, dtype_code(q), ws_ptr, ws_bytes,
                            _stream(stream)),
           "pa_decode_append")


def prefill(out, q, key_cache, value_cache, block_tables, context_lens, query_start,
            max_query_len: int, num_kv_heads: int, scale: float, stream=None):
    """Chunked prefill: rows query_start[s]..query_start[s+1]-1 of q are the
    last tokens of sequence s and attend causally over its paged context."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if hkv != num_kv_heads:
        raise ValueError("num_kv_heads does not match the cache")
    T, hq, dq = q.shape
    if dq != d or tuple(out.shape) != (T, hq, d) or out.dtype != q.dtype or q.dtype != key_cache.dtype:
        raise ValueError("q / out must be [T, Hq, d] of the cache dtype")
    S = int(context_lens.shape[0])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or query_start.shape != (S + 1,):
        raise ValueError("block_tables [S, max_blocks], context_lens [S], query_start [S + 1]")
    _check(pa_prefill(_dev(out, "out"), _dev(q, "q"), _dev(key_cache, "key_cache"),
                      _dev(value_cache, "value_cache"),
                      _dev(block_tables, "block_tables", torch.int32, 2),
                      _dev(context_lens, "context_lens", torch.int32, 1),
                      _dev(query_start, "query_start", torch.int32, 1), int(max_query_len), hkv,
                      float(scale), S, hq, T, d, bs, int(block_tables.shape[1]), nb, dtype_code(q),
                      _stream(stream)), "pa_prefill")


PREFILL_KERNELS = {"auto": 0, "mma_sync": 1, "tcgen05": 2}


def prefill_select(kernel: str) -> None:
    """Which kernel prefill() runs, process-wide: "auto" (the tcgen05 kernel
    when q / out are 16-byte aligned and the query group is at most 128, else
    the mma.sync kernel), "mma_sync" or "tcgen05"."""
    if kernel not in PREFILL_KERNELS:
        raise ValueError(f"kernel must be one of {sorted(PREFILL_KERNELS)}")
    _check(pa_prefill_select(PREFILL_KERNELS[kernel]), "pa_prefill_select")


def decode_static_workspace(out, q, key_cache, value_cache, block_tables, context_lens,
                            num_kv_heads: int, scale: float, stream=None):
    """pa_decode without a workspace argument, for callers that cannot allocate
    device memory (their memory is reserved up front by their own pools, or
    the call sits in a loop that must not call cudaMalloc).  The split-context
    scratch is a fixed array of STATIC_WORKSPACE_BYTES inside the library;
    larger problems raise PagedError(PA_ERR_WORKSPACE).  Calls sharing the
    array must not overlap on the GPU."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if hkv != num_kv_heads:
        raise ValueError("num_kv_heads does not match the cache")
    S, hq, dq = q.shape
    if dq != d or tuple(out.shape) != (S, hq, d) or out.dtype != q.dtype or q.dtype != key_cache.dtype:
        raise ValueError("q / out must be [S, Hq, d] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    _check(pa_decode_static_workspace(
        _dev(out, "out"), _dev(q, "q"), _dev(key_cache, "key_cache"),
        _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables", torch.int32, 2),
        _dev(context_lens, "context_lens", torch.int32, 1), hkv, float(scale), S, hq, d, bs,
        int(block_tables.shape[1]), nb, dtype_code(q), _stream(stream)),
        "pa_decode_static_workspace")


def copy_blocks(key_cache, value_cache, src_dst_pairs, stream=None):
    """Copy whole blocks src -> dst for each row of src_dst_pairs [P][2] (int32)."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    P = int(src_dst_pairs.shape[0]) if src_dst_pairs.numel() else 0
    if P and tuple(src_dst_pairs.shape) != (P, 2):
        raise ValueError("src_dst_pairs must be [P, 2]")
    ptr = _dev(src_dst_pairs, "src_dst_pairs", torch.int32) if P else None
    _check(pa_copy_blocks(_dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"), ptr, P,
                          hkv, d, bs, nb, dtype_code(key_cache), _stream(stream)), "pa_copy_blocks")


def swap_blocks(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache, src_dst_pairs,
                stream=None):
    """Copy whole blocks between two caches (device or pinned host tensors);
    src_dst_pairs is a host int32 array [P][2]."""
    snb, hkv, bs, d = _cache_shape(src_key_cache, src_value_cache)
    dnb, hkv2, bs2, d2 = _cache_shape(dst_key_cache, dst_value_cache)
    if (hkv, bs, d) != (hkv2, bs2, d2) or src_key_cache.dtype != dst_key_cache.dtype:
        raise ValueError("source and destination caches must have the same block shape")
    for t, n in ((src_key_cache, "src_key_cache"), (src_value_cache, "src_value_cache"),
                 (dst_key_cache, "dst_key_cache"), (dst_value_cache, "dst_value_cache")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int32).reshape(-1, 2)
    _check(pa_swap_blocks(ctypes.c_void_p(src_key_cache.data_ptr()),
                          ctypes.c_void_p(src_value_cache.data_ptr()), snb,
                          ctypes.c_void_p(dst_key_cache.data_ptr()),
                          ctypes.c_void_p(dst_value_cache.data_ptr()), dnb,
                          pairs.ctypes.data if len(pairs) else None, int(len(pairs)), hkv, d, bs,
                          dtype_code(src_key_cache), _stream(stream)), "pa_swap_blocks")


def selftest_wait_timeout(timeout_ns: int = 1_000_000, stream=None):
    """Run the bounded-wait failure path once on the device (see pa_api.h)."""
    _check(pa_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "pa_selftest_wait_timeout")


def get_error(stream=None):
    """Synchronise the stream, return (status, PA_DEVERR_* bits) and clear them."""
    bits = ctypes.c_uint32(0)
    rc = pa_get_error(_stream(stream), ctypes.byref(bits))
    return rc, int(bits.value)


# ---------------------------------------------------------------- host allocator
class BlockAllocator:
    """Host block allocator (free list, refcounts, copy-on-write) of libpa.so."""

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE):
        self._destroy = pa_alloc_destroy  # kept: module globals may be gone at exit
        self._h = pa_alloc_create(num_blocks, block_size)
        if not self._h:
            raise ValueError("bad pool size")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._destroy(h)
            self._h = None

    def add_seq(self, seq_id: int, num_tokens: int):
        _check(pa_alloc_add_seq(self._h, seq_id, num_tokens), "pa_alloc_add_seq")

    def enable_prefix_caching(self, enable: bool = True):
        _check(pa_alloc_enable_prefix_caching(self._h, int(bool(enable))),
               "pa_alloc_enable_prefix_caching")

    def add_seq_tokens(self, seq_id: int, tokens) -> int:
        """Add a prompt by its token ids; returns how many leading tokens are
        already cached (their K/V need not be written again)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        cached = _i32(0)
        _check(pa_alloc_add_seq_tokens(self._h, seq_id, t.ctypes.data if t.size else None,
                                       int(t.size), ctypes.byref(cached)), "pa_alloc_add_seq_tokens")
        return cached.value

    def fork(self, parent_id: int, child_id: int):
        _check(pa_alloc_fork(self._h, parent_id, child_id), "pa_alloc_fork")

    def append_slot(self, seq_id: int):
        """-> (slot, (cow_src, cow_dst)) with (-1, -1) when no copy is needed."""
        slot, src, dst = _i64(), _i32(), _i32()
        _check(pa_alloc_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                    ctypes.byref(dst)), "pa_alloc_append_slot")
        return slot.value, (src.value, dst.value)

    def append_slots(self, seq_ids):
        """-> (slots int64 [n], copy pairs int32 [P][2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = int(ids.shape[0])
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(n, 1), 2), np.int32)
        npairs = _i32(0)
        _check(pa_alloc_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                     pairs.ctypes.data, ctypes.byref(npairs)), "pa_alloc_append_slots")
        return slots, pairs[:npairs.value].copy()

    def free_seq(self, seq_id: int):
        _check(pa_alloc_free_seq(self._h, seq_id), "pa_alloc_free_seq")

    def num_tokens(self, seq_id: int) -> int:
        n = pa_alloc_num_tokens(self._h, seq_id)
        _check(min(n, 0), "pa_alloc_num_tokens")
        return n

    def block_table(self, seq_id: int) -> np.ndarray:
        n = pa_alloc_block_table(self._h, seq_id, None, 0)
        _check(min(n, 0), "pa_alloc_block_table")
        out = np.empty(max(n, 1), np.int32)
        pa_alloc_block_table(self._h, seq_id, out.ctypes.data, n)
        return out[:n]

    def build_tables(self, seq_ids, max_blocks: int):
        """-> (tables int32 [n][max_blocks] padded with -1, context_lens int32 [n])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = int(ids.shape[0])
        tables = np.empty((n, max_blocks), np.int32)
        lens = np.empty(n, np.int32)
        _check(pa_alloc_build_tables(self._h, ids.ctypes.data, n, tables.ctypes.data, max_blocks,
                                     lens.ctypes.data), "pa_alloc_build_tables")
        return tables, lens

    def refcount(self, block: int) -> int:
        return int(pa_alloc_refcount(self._h, block))

    def stats(self) -> dict:
        st = AllocStats()
        _check(pa_alloc_get_stats(self._h, ctypes.byref(st)), "pa_alloc_get_stats")
        return {name: getattr(st, name) for name, _ in AllocStats._fields_}


def simulate_continuous_batching(num_blocks: int, max_num_seqs: int, prompt_lens, output_lens,
                                 block_size: int = BLOCK_SIZE, max_steps: int = 10_000_000) -> dict:
    """Iteration-level scheduling over the allocator; returns the stats dict."""
    pl = np.ascontiguousarray(prompt_lens, dtype=np.int32)
    ol = np.ascontiguousarray(output_lens, dtype=np.int32)
    st = SimStats()
    _check(pa_sim_continuous_batching(num_blocks, block_size, max_num_seqs,
                                      pl.ctypes.data if pl.size else None,
                                      ol.ctypes.data if ol.size else None, int(pl.size),
                                      max_steps, ctypes.byref(st)), "pa_sim_continuous_batching")
    return {name: getattr(st, name) for name, _ in SimStats._fields_}


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    return int(pa_kv_bytes_per_token(layers, kv_heads, head_dim, dtype_bytes))


def pool_bytes(gpu_bytes: float, weight_bytes: float, utilization: float) -> float:
    return float(pa_pool_bytes(gpu_bytes, weight_bytes, utilization))


def pool_num_blocks(pool_bytes_: float, layers: int, kv_heads: int, head_dim: int,
                    block_size: int = BLOCK_SIZE, dtype_bytes: int = 2) -> int:
    return int(pa_pool_num_blocks(pool_bytes_, layers, kv_heads, head_dim, block_size, dtype_bytes))
