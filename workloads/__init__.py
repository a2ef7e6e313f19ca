"""Seeded synthetic inputs for the paged decode workloads.

This module holds random draws only: context lengths, the N(0,1) values of
q / k / v / cache contents rounded to the storage type, random orders of
physical block ids, and per-branch token counts.  It contains none of the
attention, scatter, copy or allocation arithmetic, so both the CUDA path and
the CPU oracle can take their inputs from here without sharing any of the
method's code.

Draw order for every workload (``numpy.random.default_rng(seed)``, seed 0
unless a test says otherwise):

1. context lengths (``draw_context_lens``),
2. the order in which physical block ids are handed out
   (``draw_block_order``),
3. q, then the new-token k, then the new-token v (``draw_values``),
4. the key cache contents, then the value cache contents.

Values are drawn as float32 N(0, 1) and rounded to nearest-even into the
16-bit storage type; both sides consume the rounded bit patterns.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

F16 = 0
BF16 = 1
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic decode workload."""

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: int
    layers: int
    lens: tuple  # ("uniform", lo, hi) or ("lognormal", mu, sigma, lo, hi)
    pool_factor: float = 1.1
    pool_blocks: int = 0  # fixed pool size (0: pool_factor x need)
    fragmented: bool = False
    # parallel sampling: prompts x branches; each branch adds U{0..own_max}
    prompts: int = 0
    branches: int = 0
    prompt_len: int = 0
    own_max: int = 0
    # chunked prefill: every sequence's last `chunk` tokens are the query chunk
    chunk: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    # 4 seqs, 4 q = 4 kv heads, d 64, fp16, ctx U{1..64}, 64-block pool
    "tiny": Workload("tiny", 4, 4, 4, 64, 16, F16, 1, ("uniform", 1, 64), pool_blocks=64),
    # Llama-7B decode step: 64 seqs, 32/32 heads, d 128, fp16, 32 layers
    "llama7b": Workload("llama7b", 64, 32, 32, 128, 16, F16, 32, ("lognormal", 6.0, 0.8, 16, 2048)),
    # Llama-13B decode: 256 seqs, 40/40 heads, fragmented pool, 40 layers
    "llama13b": Workload("llama13b", 256, 40, 40, 128, 16, F16, 40, ("lognormal", 6.5, 0.9, 16, 4096),
                         fragmented=True),
    # Llama-3.1-8B GQA long context: 32 seqs, 32 q / 8 kv heads, bf16
    "gqa_long": Workload("gqa_long", 32, 32, 8, 128, 16, BF16, 32, ("uniform", 8192, 32768)),
    # parallel sampling: 32 prompts x 4 branches of a 1000-token prompt
    "cow": Workload("cow", 128, 32, 32, 128, 16, BF16, 32, ("fixed", 1000), prompts=32, branches=4,
                    prompt_len=1000, own_max=256),
    # chunked prefill: 16 seqs x 512-token chunks (an 8192-token step budget)
    # over contexts U{512..4096}, Llama-3.1-8B shape (32 q / 8 kv heads, bf16)
    "prefill": Workload("prefill", 16, 32, 8, 128, 16, BF16, 32, ("uniform", 512, 4096), chunk=512),
}


def rng_for(seed: int = 0) -> np.random.Generator:
    return np.random.default_rng(seed)


def draw_context_lens(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """Context length per sequence (int32), drawn per the workload's recipe."""
    kind = w.lens[0]
    if kind == "uniform":
        lo, hi = w.lens[1], w.lens[2]
        return rng.integers(lo, hi + 1, size=w.num_seqs, dtype=np.int64).astype(np.int32)
    if kind == "lognormal":
        mu, sigma, lo, hi = w.lens[1:]
        x = rng.lognormal(mu, sigma, size=w.num_seqs)
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    if kind == "fixed":
        return np.full(w.num_seqs, w.lens[1], dtype=np.int32)
    raise ValueError(kind)


def draw_branch_tokens(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """Own-token count per branch, U{0..own_max} (parallel-sampling workload)."""
    return rng.integers(0, w.own_max + 1, size=w.prompts * w.branches, dtype=np.int64).astype(np.int32)


def draw_block_order(num_blocks: int, rng: np.random.Generator) -> np.ndarray:
    """A random permutation of physical block ids 0..num_blocks-1 (int32)."""
    return rng.permutation(num_blocks).astype(np.int32)


def round_to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """float32 -> uint16 bit patterns of fp16 / bf16, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def draw_values(rng: np.random.Generator, shape, dtype: int, chunk: int = 1 << 24) -> np.ndarray:
    """N(0, 1) float32 draws rounded to the storage type, as uint16 bits."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = round_to_bits(rng.standard_normal(m, dtype=np.float32), dtype)
    return out.reshape(shape)


def blocks_needed(lens: np.ndarray, block_size: int) -> int:
    return int(sum((int(n) + block_size - 1) // block_size for n in lens))


def pool_size(w: Workload, lens: np.ndarray) -> int:
    """Physical blocks in the pool: fixed, or pool_factor x the blocks the lengths need."""
    if w.pool_blocks:
        return w.pool_blocks
    return int(math.ceil(w.pool_factor * blocks_needed(lens, w.block_size)))


def scaled(w: Workload, **changes) -> Workload:
    """The same workload with some fields changed (smaller parity cases)."""
    return dataclasses.replace(w, **changes)
