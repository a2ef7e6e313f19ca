"""Decode batches built by the host block allocator.

Each builder takes a workload shape and its seeded draws (context lengths,
the order in which free blocks were returned, branch lengths), drives the
C++ allocator of libpa.so through the calls a serving loop makes (claim a
prompt's blocks, fork branches, append one slot per sequence), and returns
the block tables, context lengths, slots and copy-on-write pairs the kernels
consume.

A scattered pool is made the way a long-running server gets one: every block
is handed out and then freed in a random order, so the free list - and hence
each new sequence's table - follows that order ("Inside vLLM: How
PagedAttention Changes Python LLM Inference at the Systems Level", section
"The Fragmentation Problem": freed blocks end up scattered).
"""
from __future__ import annotations

import dataclasses

import numpy as np

import workloads as wl

from . import BLOCK_SIZE, BlockAllocator


@dataclasses.dataclass
class Batch:
    alloc: BlockAllocator
    seq_ids: np.ndarray       # int64 [S]
    tables: np.ndarray        # int32 [S][max_blocks], -1 padded
    context_lens: np.ndarray  # int32 [S], new token included
    slots: np.ndarray         # int64 [S], slot of each sequence's new token
    pairs: np.ndarray         # int32 [P][2], copy-on-write copies to do first
    num_blocks: int

    @property
    def max_blocks(self) -> int:
        return int(self.tables.shape[1])


def scattered_allocator(num_blocks: int, free_order: np.ndarray) -> BlockAllocator:
    """A pool whose free list hands blocks out in `free_order`."""
    a = BlockAllocator(num_blocks, BLOCK_SIZE)
    for b in range(num_blocks):
        a.add_seq(-1 - b, 1)  # claims block b (fresh pools hand out 0, 1, 2, ...)
    for b in free_order:
        a.free_seq(-1 - int(b))
    return a


def decode_batch(w: wl.Workload, lens: np.ndarray, free_order: np.ndarray, num_blocks: int,
                 max_blocks: int | None = None) -> Batch:
    """Sequences of lens[s] tokens: a prompt of lens[s] - 1 tokens plus one new token."""
    a = scattered_allocator(num_blocks, free_order)
    ids = np.arange(len(lens), dtype=np.int64)
    for s, L in zip(ids, lens):
        a.add_seq(int(s), int(L) - 1)
    slots, pairs = a.append_slots(ids)
    if max_blocks is None:
        max_blocks = max(1, (int(max(lens)) + BLOCK_SIZE - 1) // BLOCK_SIZE)
    tables, ctx = a.build_tables(ids, max_blocks)
    return Batch(a, ids, tables, ctx, slots, pairs, num_blocks)


def max_blocks_for(w: wl.Workload) -> int:
    """Table width: the workload's largest possible context in blocks."""
    hi = w.lens[-1] if w.lens[0] != "fixed" else w.prompt_len + w.own_max + 1
    return (int(hi) + BLOCK_SIZE - 1) // BLOCK_SIZE


def cow_pool_blocks(w: wl.Workload) -> int:
    prompt_blocks = (w.prompt_len + BLOCK_SIZE - 1) // BLOCK_SIZE
    n = w.prompts * w.branches
    per_branch = (w.own_max + BLOCK_SIZE - 1) // BLOCK_SIZE + 2
    return int(np.ceil(w.pool_factor * (w.prompts * prompt_blocks + n * per_branch)))


class ForkedBatch:
    """Parallel sampling: each prompt forked into `branches` sequences that
    share its blocks; every step appends one token to each live branch, and a
    branch that writes into a still-shared block gets its own copy first
    ("Inside vLLM ...", section "Copy-on-Write Makes Beam Search Cheap")."""

    def __init__(self, w: wl.Workload, own_tokens: np.ndarray, free_order: np.ndarray,
                 num_blocks: int):
        self.w = w
        self.own = np.asarray(own_tokens, dtype=np.int64)
        self.alloc = scattered_allocator(num_blocks, free_order)
        self.num_blocks = num_blocks
        self.max_blocks = max_blocks_for(w)
        n = w.prompts * w.branches
        self.seq_ids = np.arange(n, dtype=np.int64)
        for p in range(w.prompts):
            parent = p * w.branches
            self.alloc.add_seq(parent, w.prompt_len)
            for b in range(1, w.branches):
                self.alloc.fork(parent, parent + b)
        self.step_index = 0

    @property
    def num_steps(self) -> int:
        return int(self.own.max()) + 1 if len(self.own) else 0

    def step(self) -> Batch:
        """Append one token to every live branch and return that step's batch.

        Branch b generates 1 + own_tokens[b] tokens: every branch writes at
        step 0 (the step where the shared last prompt block diverges), and
        branch b is live at step k while k <= own_tokens[b]."""
        k = self.step_index
        live = self.seq_ids[self.own >= k]
        slots, pairs = self.alloc.append_slots(live)
        tables, ctx = self.alloc.build_tables(live, self.max_blocks)
        self.step_index += 1
        return Batch(self.alloc, live, tables, ctx, slots, pairs, self.num_blocks)
