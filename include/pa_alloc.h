/*
 * pa_alloc.h - host-side block allocator for the paged KV cache (libpa.so).
 *
 * Sources:
 *  - "Inside vLLM: How PagedAttention Changes Python LLM Inference at the
 *    Systems Level", section "PagedAttention: What the OS Figured Out Decades
 *    Ago": the pool is cut into fixed-size blocks; each sequence has a block
 *    table from logical block index to physical block; blocks are claimed as
 *    generation proceeds and released as soon as a sequence finishes.
 *  - same page, section "Copy-on-Write Makes Beam Search Cheap": branches of
 *    one prompt share its blocks by reference count; only a branch that
 *    writes into a shared block gets a copy of that block, the rest stays
 *    shared.
 *  - same page, section "PagedAttention in a Python RAG Application", and its
 *    question "How does prefix caching work in vLLM and when does it actually
 *    help?": the content of each block is hashed, and a request whose prefix
 *    matches reuses the cached physical blocks instead of recomputing them.
 *  - same page, section "Python LLM Inference Optimization with vLLM:
 *    Parameters That Actually Matter": the block pool takes a fraction
 *    (gpu_memory_utilization) of the memory left after the weights; under
 *    memory pressure sequences are swapped out or recomputed.
 *  - "PagedAttention in vLLM: a throughput settings guide", section
 *    "Continuous Batching Keeps the GPU Busy": the scheduler revisits the
 *    batch every step, and too many sequences for the KV budget cause
 *    preemption.
 *  - "vLLM PagedAttention: reducing KV cache memory waste", section "How
 *    PagedAttention Works": only a sequence's last block can be partly
 *    empty, so waste is bounded by one block per sequence.
 *  - same page, section "Why KV Cache Dominates GPU Memory", and "Inside
 *    vLLM ...", section "The Real Reason Your GPU Memory Is Full When It
 *    Isn't": KV bytes = 2 x layers x tokens x hidden x bytes per element.
 *
 * The allocator is plain host C++ (no CUDA call).  It is not thread-safe:
 * one thread drives one allocator.  Free blocks are handed out first in,
 * first out: a freshly created pool hands out 0, 1, 2, ...; a block freed
 * later goes to the back of the queue.  Every call that fails leaves the
 * allocator unchanged.
 */
#ifndef PA_ALLOC_H
#define PA_ALLOC_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_alloc pa_alloc;

typedef struct {
    int64_t num_blocks;     /* pool size */
    int64_t free_blocks;    /* on the free list */
    int64_t used_blocks;    /* refcount > 0 */
    int64_t shared_blocks;  /* refcount > 1 */
    int64_t num_seqs;       /* live sequences */
    int64_t logical_tokens; /* sum of the sequences' token counts */
    int64_t logical_blocks; /* sum of the sequences' table lengths */
    int64_t filled_slots;   /* slots of used blocks that hold a token */
    int64_t cow_copies;     /* copy pairs emitted since creation */
    int64_t cached_blocks;  /* full blocks findable by content (prefix caching) */
    int64_t prefix_query_blocks; /* full prompt blocks looked up since creation */
    int64_t prefix_hit_blocks;   /* of those, found in the cache and shared */
    double usage;           /* used_blocks / num_blocks */
    double waste;           /* 1 - filled_slots / (used_blocks * block_size) */
    double sharing_saving;  /* 1 - used_blocks / logical_blocks */
} pa_alloc_stats;

/* New pool of num_blocks blocks of block_size tokens, all free.  NULL on a
 * non-positive size or out of host memory. */
pa_alloc *pa_alloc_create(int32_t num_blocks, int32_t block_size);
void pa_alloc_destroy(pa_alloc *a);

/* Register sequence seq_id holding num_tokens tokens (a prompt) and claim
 * ceil(num_tokens / block_size) blocks for it.  PA_ERR_INVALID_ARG if the id
 * exists or num_tokens < 0; PA_ERR_NO_BLOCKS (nothing claimed) if the free
 * list is too short. */
int pa_alloc_add_seq(pa_alloc *a, int64_t seq_id, int32_t num_tokens);

/* child_id becomes a branch of parent_id: same tokens, same physical blocks,
 * every block's refcount + 1.  No block is claimed. */
int pa_alloc_fork(pa_alloc *a, int64_t parent_id, int64_t child_id);

/* Make room for one more token of seq_id at position p = its token count.
 * If p starts a new block, claim one and append it to the table.  Else, if
 * the last block is shared (refcount > 1), claim a fresh block, drop one
 * reference to the shared one, put the fresh one in the table and report
 * (*cow_src, *cow_dst) = (shared, fresh): the caller must copy that block
 * (pa_copy_blocks) before writing the token.  Otherwise the token goes into
 * the last block in place.  *cow_src = *cow_dst = -1 when no copy is needed.
 * *slot = table[p / block_size] * block_size + p % block_size.  The token
 * count becomes p + 1. */
int pa_alloc_append_slot(pa_alloc *a, int64_t seq_id, int64_t *slot, int32_t *cow_src,
                         int32_t *cow_dst);

/* pa_alloc_append_slot for n sequences in order.  slots[i] receives the
 * slot of seq_ids[i]; copy pairs are appended to pairs ([n][2] capacity) and
 * counted in *num_pairs.  On PA_ERR_NO_BLOCKS the sequences before the
 * failing one keep their new slot; *num_pairs counts their pairs. */
int pa_alloc_append_slots(pa_alloc *a, const int64_t *seq_ids, int32_t n, int64_t *slots,
                          int32_t *pairs, int32_t *num_pairs);

/* Drop seq_id: every block's refcount - 1; blocks reaching 0 go to the back
 * of the free list at once. */
int pa_alloc_free_seq(pa_alloc *a, int64_t seq_id);

/* Token count of seq_id, or PA_ERR_INVALID_ARG if unknown. */
int32_t pa_alloc_num_tokens(const pa_alloc *a, int64_t seq_id);

/* Copy seq_id's block table into out (at most cap entries); returns its
 * length, or PA_ERR_INVALID_ARG. */
int32_t pa_alloc_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int32_t cap);

/* Padded table matrix for a batch: row i of tables ([n][max_blocks], host)
 * receives seq_ids[i]'s table followed by -1s; context_lens[i] its token
 * count.  PA_ERR_INVALID_ARG if a table is longer than max_blocks. */
int pa_alloc_build_tables(const pa_alloc *a, const int64_t *seq_ids, int32_t n, int32_t *tables,
                          int32_t max_blocks, int32_t *context_lens);

/* Automatic prefix caching on (enable != 0) or off.  When on, every full
 * block of a prompt added with pa_alloc_add_seq_tokens is registered under a
 * chain hash of its token ids and of all the tokens before it (64-bit FNV-1a
 * over the previous block's hash and this block's ids).  A registered block
 * keeps its place in the cache after its last holder frees it: it goes to
 * the back of the free list and stays findable until the free list hands it
 * out again (first in, first out = least recently released first).  Turning
 * caching off forgets every registration. */
int pa_alloc_enable_prefix_caching(pa_alloc *a, int32_t enable);

/* pa_alloc_add_seq for a prompt whose token ids are known.  With prefix
 * caching on, the longest run of leading full blocks whose chain hash and
 * token ids match registered blocks is shared (refcount + 1; a cached block
 * on the free list leaves it) instead of claimed, and the blocks claimed for
 * the remaining full blocks are registered.  *num_cached_tokens receives the
 * number of leading tokens whose K/V are already in the cache (a multiple of
 * block_size); the caller writes K/V only for the tokens after them.  The
 * partly filled last block is never shared.  Without prefix caching this is
 * pa_alloc_add_seq with *num_cached_tokens = 0.  PA_ERR_NO_BLOCKS (nothing
 * changed) if the free list cannot serve the blocks that are not cached. */
int pa_alloc_add_seq_tokens(pa_alloc *a, int64_t seq_id, const int32_t *tokens,
                            int32_t num_tokens, int32_t *num_cached_tokens);

/* Current reference count of a physical block (0 = free), or -1. */
int32_t pa_alloc_refcount(const pa_alloc *a, int32_t block);

int pa_alloc_get_stats(const pa_alloc *a, pa_alloc_stats *out);

/* Result of pa_sim_continuous_batching. */
typedef struct {
    int64_t steps;            /* decoding steps simulated */
    int64_t tokens_generated; /* new tokens produced (each counted once) */
    int64_t preemptions;      /* sequences evicted for lack of blocks */
    int64_t admitted;         /* admissions, re-admissions after preemption included */
    int64_t finished;         /* requests that produced all their tokens */
    int64_t rejected;         /* requests that could never fit in the pool */
    double mean_usage;        /* mean fraction of pool blocks in use after a step */
    double max_usage;
    double mean_running;      /* mean sequences running after a step */
} pa_sim_stats;

/* Iteration-level scheduling ("continuous batching") on a pool of
 * num_blocks blocks.  Request r has prompt_lens[r] prompt tokens and wants
 * output_lens[r] >= 1 new tokens; all requests wait in a first-in-first-out
 * queue at step 0.  Every step: (1) while fewer than max_num_seqs run, the
 * queue's head is admitted if the pool can hold its prompt plus the tokens
 * it generated before any preemption (that prefix is recomputed); (2) every
 * running sequence appends one token; if the pool is out of blocks, the
 * latest-admitted running sequence is preempted (its blocks freed at once,
 * it returns to the front of the queue), repeatedly, until the append fits
 * or the sequence itself was preempted; a sequence that produced all its
 * tokens frees its blocks at once.  Requests whose whole life exceeds the
 * pool are rejected up front.  Stops when every request finished or after
 * max_steps. */
int pa_sim_continuous_batching(int32_t num_blocks, int32_t block_size, int32_t max_num_seqs,
                               const int32_t *prompt_lens, const int32_t *output_lens,
                               int32_t num_requests, int64_t max_steps, pa_sim_stats *out);

/* KV bytes one token occupies across all layers: 2 x layers x kv_heads x
 * head_dim x dtype_bytes (K and V). */
int64_t pa_kv_bytes_per_token(int32_t layers, int32_t kv_heads, int32_t head_dim,
                              int32_t dtype_bytes);

/* Pool bytes for a GPU: utilization x (gpu_bytes - weight_bytes), 0 if the
 * weights do not fit. */
double pa_pool_bytes(double gpu_bytes, double weight_bytes, double utilization);

/* Blocks that fit in pool_bytes for a model of that shape:
 * floor(pool_bytes / (block_size x pa_kv_bytes_per_token(...))). */
int64_t pa_pool_num_blocks(double pool_bytes, int32_t layers, int32_t kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t dtype_bytes);

#ifdef __cplusplus
}
#endif

#endif /* PA_ALLOC_H */
