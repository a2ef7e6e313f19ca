"""fp64 CPU oracle for paged decode attention, scatter-write and block copy.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  It shares no code
with the CUDA library and imports nothing from it; the two meet only in the
seeded inputs of the ``workloads`` module.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64, OpenMP over
independent (sequence, head) rows).  This module compiles it with gcc on
first use and marshals numpy arrays into it.

Every function is pinned by ``tests/test_oracle_pins.py`` against things
other than itself: exhaustive fp16 / bf16 widening against numpy, torch's
fp64 scaled-dot-product attention on densely stored K/V (with a causal mask
for chunked prefill), closed forms (one token, identical keys, constant
values, two-token logistic weights) and invariants (physical block
placement, split-range merge, a one-token chunk equals decode).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into oracle/_build/liboracle.so (gcc, -fopenmp)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load(path: str | None = None):
    global _lib
    with _lock:
        if _lib is None or path is not None:
            lib = ctypes.CDLL(path or build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_to_f64.restype = f64
            lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_f64.restype = f64
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64]
            lib.oracle_reshape_and_cache.restype = i64
            lib.oracle_copy_blocks.argtypes = [P, P, P, i32, i32, i32, i32, i64]
            lib.oracle_copy_blocks.restype = i64
            lib.oracle_decode_range.argtypes = [P, P, P, P, P, P, i32, P, i32, i32, i32, i32, i32,
                                                f64, i32, P, i32, i32, i32]
            lib.oracle_decode_range.restype = None
            lib.oracle_lse_merge.argtypes = [P, P, P, i64, i32, i32]
            lib.oracle_lse_merge.restype = None
            lib.oracle_prefill.argtypes = [P, P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, f64,
                                           i32]
            lib.oracle_prefill.restype = None
            if path is not None:
                return lib
            _lib = lib
    return _lib


def _swap_library(path: str | None):
    """Point this module at another build of the oracle (None: the normal one).

    Used only by the mutation test, which compiles copies of pa_oracle.c with
    one planted mistake each and checks that the pins reject every copy."""
    global _lib
    lib = _load(path) if path is not None else None
    with _lock:
        _lib = lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _req(a, dtype) -> np.ndarray:
    out = np.ascontiguousarray(a, dtype=dtype)
    return out


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def widen(bits: np.ndarray, dtype: int) -> np.ndarray:
    """fp16 / bf16 bit patterns -> float64, element by element in C."""
    lib = _load()
    fn = lib.oracle_f16_to_f64 if dtype == F16 else lib.oracle_bf16_to_f64
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([fn(int(b)) for b in flat], dtype=np.float64).reshape(np.shape(bits))


def reshape_and_cache(k, v, key_cache: np.ndarray, value_cache: np.ndarray, slot_mapping) -> int:
    """Scatter each token's K/V into its slot, in place on the uint16 caches.

    k, v: [T][Hkv][d] uint16; caches: [NB][Hkv][bs][d] uint16; slot_mapping [T].
    Returns the number of out-of-range slots skipped."""
    k = _req(k, np.uint16)
    v = _req(v, np.uint16)
    slots = _req(slot_mapping, np.int64)
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    assert key_cache.dtype == np.uint16 and value_cache.dtype == np.uint16
    nb, hkv, bs, d = key_cache.shape
    return int(_load().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(key_cache), _ptr(value_cache),
                                                _ptr(slots), int(slots.shape[0]), hkv, d, bs, nb))


def copy_blocks(key_cache: np.ndarray, value_cache: np.ndarray, pairs) -> int:
    """Copy block src -> dst (all heads, K and V) for each pair, in place."""
    pairs = _req(pairs, np.int32).reshape(-1, 2)
    nb, hkv, bs, d = key_cache.shape
    return int(_load().oracle_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(pairs),
                                          int(pairs.shape[0]), hkv, d, bs, nb))


def decode_range(q, key_cache, value_cache, block_tables, context_lens, num_kv_heads: int,
                 scale: float, dtype: int, t0: int = 0, t1: int = -1, seqs=None):
    """Attention of each (seq, q head) over tokens [t0, t1) of its context.

    Returns (out [S'][Hq][d] float64, lse [S'][Hq] float64) where S' are the
    selected sequences (all by default) and lse = log sum_j exp(scale q.k_j)."""
    q = _req(q, np.uint16)
    kc = _req(key_cache, np.uint16)
    vc = _req(value_cache, np.uint16)
    tables = _req(block_tables, np.int32)
    lens = _req(context_lens, np.int32)
    S, Hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    assert d2 == d and hkv == num_kv_heads and Hq % hkv == 0
    sel = None if seqs is None else _req(seqs, np.int32)
    ns = S if sel is None else int(sel.shape[0])
    out = np.zeros((ns, Hq, d), dtype=np.float64)
    lse = np.zeros((ns, Hq), dtype=np.float64)
    _load().oracle_decode_range(_ptr(out), _ptr(lse), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                                int(tables.shape[1]), _ptr(lens), S, Hq, hkv, d, bs, float(scale),
                                int(dtype), _ptr(sel), ns, int(t0), int(t1))
    return out, lse


def decode(q, key_cache, value_cache, block_tables, context_lens, num_kv_heads: int, scale: float,
           dtype: int, seqs=None) -> np.ndarray:
    """softmax(scale q K^T) V per (seq, q head) over the whole paged context, fp64."""
    return decode_range(q, key_cache, value_cache, block_tables, context_lens, num_kv_heads,
                        scale, dtype, 0, -1, seqs)[0]


def prefill(q, key_cache, value_cache, block_tables, context_lens, query_start, num_kv_heads: int,
            scale: float, dtype: int) -> np.ndarray:
    """Chunked prefill: query rows query_start[s]..query_start[s+1]-1 are the
    last tokens of sequence s and attend causally over its paged context.
    q [T][Hq][d] bits -> out [T][Hq][d] float64."""
    q = _req(q, np.uint16)
    kc = _req(key_cache, np.uint16)
    vc = _req(value_cache, np.uint16)
    tables = _req(block_tables, np.int32)
    lens = _req(context_lens, np.int32)
    qs = _req(query_start, np.int32)
    T, Hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    assert d2 == d and hkv == num_kv_heads and Hq % hkv == 0 and qs[-1] == T
    out = np.zeros((T, Hq, d), dtype=np.float64)
    _load().oracle_prefill(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                           int(tables.shape[1]), _ptr(lens), _ptr(qs), int(lens.shape[0]), Hq, hkv,
                           d, bs, float(scale), int(dtype))
    return out


def lse_merge(o_parts: np.ndarray, lse_parts: np.ndarray) -> np.ndarray:
    """Merge per-range results: o_parts [R][P][d], lse_parts [R][P] -> [R][d]."""
    o = _req(o_parts, np.float64)
    lse = _req(lse_parts, np.float64)
    R, P, d = o.shape
    out = np.zeros((R, d), dtype=np.float64)
    _load().oracle_lse_merge(_ptr(out), _ptr(o), _ptr(lse), R, P, d)
    return out
