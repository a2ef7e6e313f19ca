"""Test-side construction of paged problems from seeded dense draws.

Dense K/V rows are drawn per sequence straight from the generators, then
placed into a pool through a block table; this lets the oracle's gather be
checked against attention on the dense rows, which never passed through the
pool.  Nothing here calls the oracle or the CUDA library.
"""
from __future__ import annotations

import numpy as np

import workloads as wl


class Paged:
    """A paged decode problem held as host numpy arrays (uint16 bits)."""

    def __init__(self, q, key_cache, value_cache, tables, lens, num_kv_heads, scale, dtype,
                 k_dense=None, v_dense=None):
        self.q = q
        self.key_cache = key_cache
        self.value_cache = value_cache
        self.tables = tables
        self.lens = lens
        self.num_kv_heads = num_kv_heads
        self.scale = scale
        self.dtype = dtype
        self.k_dense = k_dense
        self.v_dense = v_dense

    @property
    def block_size(self):
        return self.key_cache.shape[2]


def tables_from_order(lens, order, block_size, max_blocks=None):
    """Hand consecutive chunks of a block-id order to the sequences in turn."""
    need = [(int(n) + block_size - 1) // block_size for n in lens]
    mb = max_blocks if max_blocks is not None else max(max(need), 1)
    tables = np.full((len(lens), mb), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(need):
        tables[s, :n] = order[pos:pos + n]
        pos += n
    return tables


def make_paged(rng, num_seqs, num_q_heads, num_kv_heads, head_dim, lens, num_blocks, dtype,
               block_size=16, scale=None, max_blocks=None):
    """Seeded paged problem: dense K/V rows placed into a randomly ordered pool.

    Pool rows that no token uses keep their own N(0,1) background draws."""
    lens = np.asarray(lens, dtype=np.int32)
    lmax = max(int(lens.max()) if len(lens) else 1, 1)
    order = wl.draw_block_order(num_blocks, rng)
    q = wl.draw_values(rng, (num_seqs, num_q_heads, head_dim), dtype)
    kd = wl.draw_values(rng, (num_seqs, lmax, num_kv_heads, head_dim), dtype)
    vd = wl.draw_values(rng, (num_seqs, lmax, num_kv_heads, head_dim), dtype)
    kc = wl.draw_values(rng, (num_blocks, num_kv_heads, block_size, head_dim), dtype)
    vc = wl.draw_values(rng, (num_blocks, num_kv_heads, block_size, head_dim), dtype)
    tables = tables_from_order(lens, order, block_size, max_blocks)
    for s in range(num_seqs):
        L = int(lens[s])
        nblk = (L + block_size - 1) // block_size
        if nblk == 0:
            continue
        # [nblk*bs, H, d] -> [nblk, bs, H, d] -> [nblk, H, bs, d], then write the
        # valid rows only (the tail of the last block keeps its background).
        pad = np.zeros((nblk * block_size, num_kv_heads, head_dim), dtype=np.uint16)
        for dense, pool in ((kd, kc), (vd, vc)):
            pad[:L] = dense[s, :L]
            tiles = pad.reshape(nblk, block_size, num_kv_heads, head_dim).transpose(0, 2, 1, 3)
            ids = tables[s, :nblk]
            full = L // block_size
            pool[ids[:full]] = tiles[:full]
            if full < nblk:
                rem = L - full * block_size
                pool[ids[full], :, :rem, :] = tiles[full, :, :rem, :]
    if scale is None:
        scale = 1.0 / np.sqrt(head_dim)
    return Paged(q, kc, vc, tables, lens, num_kv_heads, float(scale), dtype, kd, vd)


def to_f64(bits, dtype):
    """Independent widening for test-side references (numpy, not the oracle)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == wl.F16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
