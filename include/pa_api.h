/*
 * pa_api.h - C ABI of the paged KV-cache decode library (libpa.so).
 *
 * The library implements the data-parallel hot path of PagedAttention on
 * NVIDIA B200 (sm_100a): writing each new token's K/V into its slot of a
 * block-paged cache, copying shared blocks on write, and single-token decode
 * attention that reaches every cached token through a per-sequence block
 * table.
 *
 * Sources of the operations (web pages on PagedAttention):
 *  - "Inside vLLM: How PagedAttention Changes Python LLM Inference at the
 *    Systems Level", section "PagedAttention: What the OS Figured Out
 *    Decades Ago": fixed-size blocks of 16 tokens, a block table mapping
 *    logical to physical blocks, non-contiguous blocks that attention sees as
 *    contiguous, new blocks appended as tokens are generated.
 *  - same page, section "Copy-on-Write Makes Beam Search Cheap": shared
 *    prefix blocks by reference count; a write into a shared block copies
 *    that block only.
 *  - "vLLM PagedAttention: reducing KV cache memory waste", section "How
 *    PagedAttention Works": blocks claimed on demand, waste only in the last
 *    block, copy-on-write on divergence.
 *  - "PagedAttention in vLLM: a throughput settings guide", section
 *    "Continuous Batching Keeps the GPU Busy": decoding is bound by memory
 *    bandwidth.
 *
 * Conventions shared by every call:
 *  - Pointers marked "device" are CUDA device addresses on the current
 *    device; "host" pointers are ordinary host memory.  The caller owns every
 *    buffer.  The library allocates no device memory: scratch (workspace) is
 *    passed in by the caller.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    except pa_get_error only enqueues work on `stream` and returns.
 *  - Element types: PA_F16 (IEEE binary16) or PA_BF16 (bfloat16), 2 bytes.
 *  - Cache layout: key_cache and value_cache are each
 *      [num_blocks][num_kv_heads][block_size][head_dim]
 *    with head_dim contiguous, so one (block, kv head) tile of block_size
 *    rows is contiguous (4 KiB at head_dim 128).  Element (b, h, o, i) is at
 *    ((b * num_kv_heads + h) * block_size + o) * head_dim + i.
 *    Both caches must start on a 16-byte boundary.
 *  - Supported shapes: block_size == 16 (PA_BLOCK_SIZE), head_dim 64 or 128,
 *    num_q_heads a multiple of num_kv_heads with at most 16 query heads per
 *    kv head, num_blocks * num_kv_heads * 16 < 2^31.  Anything else returns
 *    PA_ERR_UNSUPPORTED (or PA_ERR_INVALID_ARG for inconsistent values)
 *    before any work is enqueued.
 *  - Bad indices found on the device (a block id outside [0, num_blocks), a
 *    slot outside the pool, a context length above the table's capacity) are
 *    never dereferenced: the kernel skips the access and sets a bit in the
 *    library's device error word, which pa_get_error reads and clears.
 *  - Return value: PA_OK or a negative pa_status.  A launch failure reported
 *    by the CUDA runtime returns PA_ERR_CUDA.
 */
#ifndef PA_API_H
#define PA_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = -1,  /* null pointer, negative size, inconsistent shapes */
    PA_ERR_UNSUPPORTED = -2,  /* valid but not built: block_size, head_dim, dtype, group */
    PA_ERR_OUT_OF_RANGE = -3, /* pa_get_error: the device saw a bad index */
    PA_ERR_NO_BLOCKS = -4,    /* allocator: the free list cannot serve the request */
    PA_ERR_CUDA = -5,         /* the CUDA runtime reported an error */
    PA_ERR_WORKSPACE = -6,    /* pa_decode: workspace missing or too small */
    PA_ERR_TIMEOUT = -7       /* pa_get_error: a device wait gave up */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

#define PA_BLOCK_SIZE 16
/* Decode splits a context into partitions of this many tokens (32 blocks);
 * calls whose block tables span 16384 tokens or more use twice that. */
#ifndef PA_PARTITION_TOKENS
#define PA_PARTITION_TOKENS 512
#endif

/* Bits of the device error word (pa_get_error). */
#define PA_DEVERR_BLOCK_ID 1u    /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 2u        /* slot_mapping entry >= num_blocks * block_size */
#define PA_DEVERR_PAIR 4u        /* copy pair id outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 8u /* context_len < 0 or > max_blocks_per_seq * block_size */
#define PA_DEVERR_TIMEOUT 16u    /* a bounded wait on an async copy gave up */

/*
 * pa_reshape_and_cache - write the new tokens' K and V into their cache slots.
 *
 * Source: "Inside vLLM ...", section "PagedAttention: What the OS Figured Out
 * Decades Ago" (a sequence's tokens live in the blocks its table lists; new
 * tokens go into the table's last block, or a newly appended one).
 *
 * For each token t with slot = slot_mapping[t] >= 0:
 *   key_cache  [slot / block_size][h][slot % block_size][:] = k[t][h][:]
 *   value_cache[slot / block_size][h][slot % block_size][:] = v[t][h][:]
 * for every kv head h.  The slot of a token at position p of a sequence is
 * table[p / block_size] * block_size + p % block_size (pa_alloc_append_slot
 * returns it).  A negative slot is padding and is skipped.  A slot at or
 * beyond num_blocks * block_size is skipped and sets PA_DEVERR_SLOT.
 * The copy is bit-exact.  Two tokens with the same slot race (undefined
 * which one lands).
 *
 *   k, v          device, [num_tokens][num_kv_heads][head_dim], dtype,
 *                 contiguous, 16-byte aligned
 *   key_cache,    device, cache layout above (written in place)
 *   value_cache
 *   slot_mapping  device, int64 [num_tokens]
 */
int pa_reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int64_t num_blocks, int32_t dtype,
                         void *stream);

/*
 * pa_decode - single-token decode attention over the paged cache.
 *
 * Source: "Inside vLLM ...", section "PagedAttention: What the OS Figured Out
 * Decades Ago" (the block table makes scattered blocks look contiguous to
 * attention); "PagedAttention in vLLM: a throughput settings guide", section
 * "Continuous Batching Keeps the GPU Busy" (decode reads memory, not math).
 *
 * For sequence s with L = context_lens[s] cached tokens (the new token
 * included, written beforehand by pa_reshape_and_cache; pa_decode_append
 * does both in one launch) and query head h,
 * with G = num_q_heads / num_kv_heads and kv head g = h / G:
 *   K_j = key_cache  [block_tables[s][j / 16]][g][j % 16][:],  j < L
 *   V_j = value_cache[block_tables[s][j / 16]][g][j % 16][:]
 *   out[s][h][:] = sum_j softmax_j(scale * q[s][h] . K_j) V_j
 * q . K products accumulate in fp32 and the softmax runs in fp32; the P . V
 * product takes P rounded to dtype (tensor cores; built with PA_MHA_ON_MMA=0,
 * one query head per kv head keeps P in fp32 on CUDA cores); out is rounded
 * to dtype.
 * L == 0 gives a zero row.  Table entries past ceil(L / 16) are not read.
 *
 * Contexts longer than one partition (PA_PARTITION_TOKENS tokens, or twice
 * that when max_blocks_per_seq * 16 >= 16384) are split into partitions that
 * run in parallel and are merged by log-sum-exp; the partial results go to
 * `workspace`, which must hold pa_decode_workspace_size(...) bytes (256-byte
 * aligned) whenever max_blocks_per_seq * 16 > PA_PARTITION_TOKENS, and may be
 * NULL otherwise.  Calls that share a workspace must not overlap.
 *
 *   out           device, [num_seqs][num_q_heads][head_dim], dtype
 *   q             device, [num_seqs][num_q_heads][head_dim], dtype
 *   key_cache,    device, cache layout above (read only)
 *   value_cache
 *   block_tables  device, int32 [num_seqs][max_blocks_per_seq]
 *   context_lens  device, int32 [num_seqs]
 *   scale         multiplier of q . k (typically 1 / sqrt(head_dim))
 */
int pa_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *context_lens, int32_t num_kv_heads,
              float scale, int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
              int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_decode_append - write each sequence's new token into the cache, then
 * decode: pa_reshape_and_cache followed by pa_decode, in one launch.
 *
 * Source: the passages of pa_reshape_and_cache and pa_decode.  A decode step
 * appends one token per sequence at position L - 1 (L = context_lens[s],
 * the new token included) and attends over all L tokens; this call does
 * both, so the step needs no separate write launch.
 *
 * Equivalent to pa_reshape_and_cache(k_new, v_new, ..., slot_mapping) with
 * slot_mapping[s] = block_tables[s][(L - 1) / 16] * 16 + (L - 1) % 16,
 * followed by pa_decode(...) with the same arguments: the same cache bytes
 * afterwards, and the same outputs, bit for bit.  Sequences with L == 0
 * write nothing (zero output row).  An out-of-range block id at position
 * L - 1 writes nothing and sets PA_DEVERR_BLOCK_ID, as pa_decode reports it;
 * so does a context length beyond the table (PA_DEVERR_CONTEXT_LEN), whose
 * position L - 1 has no slot.
 * The block holding position L - 1 must belong to this sequence alone (the
 * allocator copies a shared last block before appending to it): another
 * sequence that reads it in the same call may see the slot before or after
 * the write.  Argument checks, workspace and errors are those of pa_decode.
 *
 *   k_new, v_new  device, [num_seqs][num_kv_heads][head_dim], dtype,
 *                 contiguous, 16-byte aligned (PA_ERR_INVALID_ARG otherwise)
 *   key_cache,    device, cache layout of pa_decode (one row per sequence and
 *   value_cache   kv head written, the rest read)
 */
int pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                     void *key_cache, void *value_cache, const int32_t *block_tables,
                     const int32_t *context_lens, int32_t num_kv_heads, float scale,
                     int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t block_size,
                     int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_prefill - chunked-prefill attention over the paged cache.
 *
 * Source: "PagedAttention in vLLM: a throughput settings guide", section
 * "Tuning Batching, Prefill, and Cache" (chunked prefill: a step fills its
 * token budget with chunks of prompts; each chunk attends to what is cached
 * before it).
 *
 * Sequence s owns query rows query_start[s] .. query_start[s + 1] - 1 of q;
 * they are the LAST n_s = query_start[s + 1] - query_start[s] tokens of its
 * context of L = context_lens[s] tokens, and their K/V are already in the
 * cache (written by pa_reshape_and_cache).  Query row i of s sits at position
 * p = L - n_s + i; for query head h (kv head h / G):
 *   out[row][h][:] = sum_{j <= p} softmax_j(scale * q[row][h] . K_j) V_j
 * with K_j, V_j reached through block_tables[s][j / 16] as in pa_decode.
 * fp32 softmax; the P.V product takes P in the input dtype (tensor cores).
 * n_s > L or L beyond the table sets PA_DEVERR_CONTEXT_LEN (clamped).
 *
 *   out, q        device, [num_q_tokens][num_q_heads][head_dim], dtype
 *   query_start   device, int32 [num_seqs + 1], non-decreasing, [num_seqs] =
 *                 num_q_tokens
 *   max_query_len upper bound of every n_s (sizes the grid)
 */
int pa_prefill(void *out, const void *q, const void *key_cache, const void *value_cache,
               const int32_t *block_tables, const int32_t *context_lens,
               const int32_t *query_start, int32_t max_query_len, int32_t num_kv_heads,
               float scale, int32_t num_seqs, int32_t num_q_heads, int32_t num_q_tokens,
               int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
               int64_t num_blocks, int32_t dtype, void *stream);

/*
 * pa_prefill_select - which kernel pa_prefill runs (process-wide).
 *
 *   PA_PREFILL_AUTO     the tcgen05 kernel when its conditions hold (q and
 *                       out 16-byte aligned, query group <= 128, scale > 0),
 *                       otherwise the mma.sync kernel.  The default.
 *   PA_PREFILL_MMA_SYNC always the mma.sync kernel (64 packed query rows per
 *                       CTA, warp-level tensor-core tiles, registers hold S).
 *   PA_PREFILL_TCGEN05  always the tcgen05 kernel (work items of two tiles of
 *                       128 packed query rows, walked by one persistent CTA
 *                       per SM; S, P and O in tensor memory); pa_prefill
 *                       returns PA_ERR_UNSUPPORTED when its conditions fail.
 * Both compute the same operation; results differ only by rounding order.
 * Returns PA_OK, or PA_ERR_INVALID_ARG for an unknown value.
 */
#define PA_PREFILL_AUTO 0
#define PA_PREFILL_MMA_SYNC 1
#define PA_PREFILL_TCGEN05 2
int pa_prefill_select(int32_t kernel);

/* Bytes of workspace pa_decode needs for these sizes (0 when no context can
 * exceed one partition). */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_blocks_per_seq);

/*
 * pa_decode_static_workspace - pa_decode for callers that cannot allocate.
 *
 * The paper has no counterpart for this call: it is an interface
 * convenience of this library, not a step of the method.
 *
 * pa_decode needs split-context scratch (its `workspace`) whenever a context
 * can span more than one partition.  Some callers cannot hand it over:
 *  - a serving process that reserves nearly all device memory up front for
 *    its own KV block pool and weights, so any later cudaMalloc fails or
 *    fragments that reservation;
 *  - a hot decode loop that must not call cudaMalloc, because it can
 *    synchronise the device and stall every stream;
 *  - a caller in another language that reaches this library through the C
 *    ABI and has no device allocator of its own.
 * This entry point computes exactly what pa_decode computes, with the same
 * arguments minus the workspace.  Its scratch is a fixed array of
 * PA_STATIC_WORKSPACE_BYTES in the library's device memory: every GPU that
 * loads the library holds it until the process exits.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Limits and rules:
 *  - The arguments are checked first, exactly as pa_decode checks them, so
 *    the two calls return the same status for the same arguments.  Then, if
 *    pa_decode_workspace_size(...) for these sizes exceeds
 *    PA_STATIC_WORKSPACE_BYTES, the call returns PA_ERR_WORKSPACE.  A call
 *    that returns an error enqueues nothing.
 *  - The first call on a device looks up the array's device address (once
 *    per device and CUDA context, with that device current).  Make that first
 *    call before any stream capture begins.  After a cudaDeviceReset the old
 *    address belongs to a context that no longer exists; the next call, in the
 *    new context, looks the address up again (so it is again a first call).
 *  - All calls share the one array, and it keeps the last call's contents.
 *    Nothing in it has to start at zero.  Calls that overlap on the GPU
 *    (other streams, other host threads) race on the array and give wrong
 *    results: serialise them.
 */
#define PA_STATIC_WORKSPACE_BYTES ((size_t)48 << 20)
int pa_decode_static_workspace(void *out, const void *q, const void *key_cache,
                               const void *value_cache, const int32_t *block_tables,
                               const int32_t *context_lens, int32_t num_kv_heads, float scale,
                               int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                               int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
                               int32_t dtype, void *stream);

/*
 * pa_copy_blocks - copy-on-write block copies.
 *
 * Source: "Inside vLLM ...", section "Copy-on-Write Makes Beam Search Cheap";
 * "vLLM PagedAttention: reducing KV cache memory waste", section "How
 * PagedAttention Works" (copy-on-write handles divergence of shared blocks).
 *
 * For each pair p: physical block src_dst_pairs[p][1] (every kv head, every
 * row, K and V) becomes a bit-exact copy of block src_dst_pairs[p][0].
 * Destinations must be distinct and no destination may also be a source in
 * the same call (pa_alloc_append_slot never produces such pairs); otherwise
 * the result is undefined.  A pair with an id outside [0, num_blocks) is
 * skipped and sets PA_DEVERR_PAIR.
 *
 *   src_dst_pairs  device, int32 [num_pairs][2]
 */
int pa_copy_blocks(void *key_cache, void *value_cache, const int32_t *src_dst_pairs,
                   int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   int64_t num_blocks, int32_t dtype, void *stream);

/*
 * pa_swap_blocks - move whole blocks between two caches, one of which may
 * live in page-locked host memory (swap out under memory pressure, swap back
 * in later).
 *
 * Source: "Inside vLLM ...", section "Python LLM Inference Optimization with
 * vLLM: Parameters That Actually Matter" (under memory pressure a sequence's
 * blocks can be swapped to CPU RAM; swapping keeps the KV cache but costs
 * PCIe bandwidth).
 *
 * For each pair p, block src_dst_pairs[p][1] of (dst_key_cache,
 * dst_value_cache) becomes a bit-exact copy of block src_dst_pairs[p][0] of
 * (src_key_cache, src_value_cache).  Both caches have the layout above with
 * the same num_kv_heads, head_dim and dtype; each may be device memory or
 * page-locked host memory.  The pairs are a HOST array.  When every pool is
 * device memory of the current device or mapped page-locked host memory, one
 * kernel per 2048 pairs moves the blocks (host pools through their device
 * alias, over PCIe / C2C); otherwise (pageable host memory, another device)
 * the copies are one cudaMemcpyAsync per run of consecutive source and
 * destination ids, K and V separately, and pageable memory makes them
 * synchronous.  An id out of range returns PA_ERR_OUT_OF_RANGE before
 * anything is enqueued.  Destinations must be distinct and must not
 * be sources of the same call when both caches are the same memory.
 *
 *   src_dst_pairs  host, int32 [num_pairs][2]
 */
int pa_swap_blocks(const void *src_key_cache, const void *src_value_cache, int64_t src_num_blocks,
                   void *dst_key_cache, void *dst_value_cache, int64_t dst_num_blocks,
                   const int32_t *src_dst_pairs, int32_t num_pairs, int32_t num_kv_heads,
                   int32_t head_dim, int32_t block_size, int32_t dtype, void *stream);

/*
 * pa_get_error - synchronise `stream`, then read and clear the device error
 * word (one word for the whole process and device).  *bits (host, may be
 * NULL) receives the PA_DEVERR_* bits seen since the last call.  Returns
 * PA_OK if no bit was set, PA_ERR_TIMEOUT if PA_DEVERR_TIMEOUT was set,
 * PA_ERR_OUT_OF_RANGE for any other bit, PA_ERR_CUDA if the stream failed.
 */
int pa_get_error(void *stream, uint32_t *bits);

/*
 * pa_selftest_wait_timeout - diagnostic of the failure path shared by every
 * kernel: one warp waits on an mbarrier that nothing completes, gives up
 * after timeout_ns (1 ns .. 1 s) and sets PA_DEVERR_TIMEOUT, exactly as a
 * decode or prefill CTA does when a TMA tile never lands.  A following
 * pa_get_error returns PA_ERR_TIMEOUT; the CUDA context stays usable.  It has
 * no counterpart in the pages.
 */
int pa_selftest_wait_timeout(uint64_t timeout_ns, void *stream);

/* Static description of a status code. */
const char *pa_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_API_H */
