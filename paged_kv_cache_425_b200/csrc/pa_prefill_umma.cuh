// Chunked-prefill attention on the fifth-generation tensor cores (tcgen05).
//
// Same operation as prefill_mma_kernel ("PagedAttention in vLLM: a
// throughput settings guide", the chunked-prefill passage: a sequence's new
// tokens attend causally to its whole paged context), as a Blackwell
// warp-specialised pipeline.  A work item is two query tiles of 128 packed
// rows (token i, head h of the kv head's query group -> row i * G + h) of one
// (sequence, kv head); the kernel is persistent (one CTA per SM), and each
// CTA walks its items, each over the context in tiles of 128 keys (8 blocks):
//
//  * warps 8 and 10 are the producers: warp 8 TMA-loads each item's two
//    query tiles and every key tile's K blocks, warp 10 the V blocks, into
//    two-stage rings; warp 8 owns the TMEM allocation;
//  * warp 9, one thread, issues every tcgen05.mma: S_k = Q_k K^T into query
//    tile k's 128 S columns of tensor memory, and O_k += P_k V with P_k read
//    from tensor memory (it overwrites the upper half of S_k) and V from
//    shared memory; completion is signalled with tcgen05.commit;
//  * warpgroup k (warps 4k .. 4k + 3; thread r = row r = TMEM lane r) is query
//    tile k's softmax: it reads its S row from TMEM, applies the causal mask,
//    runs the online softmax in the log2 domain, rescales O_k in TMEM when the
//    running max has grown, and writes P_k back to TMEM as 16-bit values; at
//    the end it normalises O_k and stores it.
//
// Items continue the rings, barrier phases and tensor memory of the one
// before: the next item's query tiles load once the MMAs have read the last
// ones, and its first S_k is computed while warpgroup k writes out the
// previous O_k, which the next item's first P_k V overwrites only after
// warpgroup k's next arrival.
//
// The MMA order per key tile j is S_0, S_1 | P_0 V, S_0(j+1), P_1 V, S_1(j+1):
// while warpgroup 0 turns S_0 into P_0 the tensor core computes S_1 and the
// previous tile's P_1 V, and the other way round, so the softmax of one query
// tile hides behind the other tile's GEMMs.  tcgen05.mma operations issued by
// one thread run in issue order, so S_k of tile j + 1 may overwrite P_k of
// tile j once P_k V has been issued; a commit after S_k of tile j also covers
// P_k V of tile j - 1, so O_k is settled whenever S_k is ready.
//
// The running max is only raised when a tile's max exceeds it by more than 8
// (log2 units): until then P <= 2^8, which 16-bit P and f32 sums hold as well,
// and O and l stay consistent because both use the same stale max.
//
// Shared-memory tiles are stacks of 8-row x 128-byte atoms in the TMA
// 128-byte swizzle; a 128-row tile of D columns is D / 64 chunks of 16 KiB.
// Warp 11 only completes the third warpgroup (setmaxnreg works per
// warpgroup).  Every wait is bounded; a wait that gives up raises the CTA's abort flag, the
// other roles leave their loops, in-flight copies and MMAs are waited for,
// and the tensor memory is released before the CTA exits.
#pragma once

#include "pa_exp2.cuh"
#include "pa_kernels.cuh"
#include "pa_umma.cuh"

namespace pa {

constexpr int kUmmaRows = 128;         // packed query rows per query tile (MMA M)
constexpr int kUmmaQTiles = 2;         // query tiles per CTA
constexpr int kUmmaKeys = 128;         // keys per key tile (N of Q K^T, K of P V)
constexpr int kUmmaThreads = 384;      // two softmax warpgroups + one of producer / MMA issuer
// Register split (setmaxnreg): the softmax warpgroups hold a whole S row, the
// third warpgroup needs few.  The shares add up to the launch's registers
// (384 threads x 168); the host checks the compiled count before launching,
// since a larger share than the launch holds would never be granted.
constexpr int kSoftmaxRegs = 200, kOtherRegs = 104;
constexpr int kUmmaRegsNeeded = 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs;
constexpr int kUmmaChunk = 128 * 128;  // bytes: 128 rows x 128-byte swizzled chunk
constexpr uint32_t kUmmaTmemCols = 512;
constexpr float kMaxSlack = 8.f;       // log2 growth of the max tolerated before a rescale
constexpr int kRankMax = 256;          // batches up to this size are scheduled longest first
#ifndef PA_EXP2_FMA_EVERY
#define PA_EXP2_FMA_EVERY 8
#endif
// One softmax weight pair in this many is computed on the FMA pipe
// (exp2_fma_pair) instead of the special-function unit; 0 = none.
constexpr int kExp2FmaEvery = PA_EXP2_FMA_EVERY;
constexpr int kExp2Period = kExp2FmaEvery > 0 ? kExp2FmaEvery : 1;

// Dynamic shared memory: both query tiles, two K and two V stages, and
// alignment slack.
template <int D>
constexpr int prefill_umma_smem_bytes() {
    return kUmmaQTiles * kUmmaRows * D * 2 + 4 * kUmmaKeys * D * 2 + 1024;
}

template <typename T>
struct UmmaFormat;
template <>
struct UmmaFormat<__half> {
    static constexpr uint32_t value = 0;
};
template <>
struct UmmaFormat<__nv_bfloat16> {
    static constexpr uint32_t value = 1;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Wait for phase `parity` of `bar`; give up when the CTA's abort flag is
// raised, or after kWaitTimeoutNs (then raise it and flag PA_DEVERR_TIMEOUT).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (global_timer_ns() - start > kWaitTimeoutNs) {
            flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// One work item: two query tiles of one (sequence, kv head).  Items are
// numbered (sequence rank, query tile pair from the last, kv head), longest
// context first; every role of a CTA derives the same items in the same order.
struct UmmaItem {
    int s, kvh, tile, q0, n, L, row0, rows_total, nkeys, nblk, ntiles;
    const int32_t *trow;
};

// Item i; false when it has no rows (a sequence with fewer query tokens than
// the grid was sized for) or invalid bounds (reported by `report`).
__device__ __forceinline__ bool umma_item(const PrefillArgs &a, const int *s_order, int i, int G,
                                          int rows_used, bool report, UmmaItem &it) {
    const int per_seq = a.tiles_per_seq * a.num_kv_heads;
    const int rank = i / per_seq, rem = i % per_seq;
    it.tile = a.tiles_per_seq - 1 - rem / a.num_kv_heads;
    it.kvh = rem % a.num_kv_heads;
    it.s = a.num_seqs <= kRankMax ? s_order[rank] : rank;
    it.q0 = a.query_start[it.s];
    int n = a.query_start[it.s + 1] - it.q0;
    int L = a.context_lens[it.s];
    const int cap = a.max_blocks_per_seq * kBlock;
    const bool head = it.tile == 0 && it.kvh == 0;  // one item per sequence reports
    if (it.q0 < 0 || it.q0 > a.num_q_tokens || n > a.num_q_tokens - it.q0) {
        if (report && head) flag_error(PA_DEVERR_CONTEXT_LEN);
        return false;
    }
    if (L < 0 || L > cap || n < 0 || n > L) {
        if (report && head) flag_error(PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : (L > cap ? cap : L);
        n = n < 0 ? 0 : (n > L ? L : n);
    }
    it.n = n;
    it.L = L;
    it.rows_total = n * G;
    it.row0 = it.tile * kUmmaQTiles * rows_used;
    if (it.row0 >= it.rows_total) return false;
    const int last_row = min(it.rows_total, it.row0 + kUmmaQTiles * rows_used) - 1;
    it.nkeys = L - n + last_row / G + 1;
    it.nblk = (it.nkeys + kBlock - 1) / kBlock;
    it.ntiles = (it.nkeys + kUmmaKeys - 1) / kUmmaKeys;
    it.trow = a.block_tables + (size_t)it.s * a.max_blocks_per_seq;
    return true;
}

// Item of the CTA's r-th round: rounds go over the items in order, P per
// round, alternately forwards and backwards over the CTAs (a snake), so the
// longest items of a round and the shortest of the next land on the same CTA.
__device__ __forceinline__ int umma_round_item(int r) {
    const int P = gridDim.x, c = blockIdx.x;
    return r * P + ((r & 1) ? P - 1 - c : c);
}

template <typename T, int D>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    prefill_umma_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const PrefillArgs a) {
    static_assert(D == 64 || D == 128, "head dim");
    constexpr int NCH = D / 64;                   // 128-byte chunks per row
    constexpr int QB = kUmmaRows * D * 2;         // one query tile
    constexpr int KVB = kUmmaKeys * D * 2;        // one K or V tile
    constexpr int QK_STEPS = D / 16, PV_STEPS = kUmmaKeys / 16;
    constexpr uint32_t FMT = UmmaFormat<T>::value;
    // TMEM columns: S_k at 128 k (P_k over its upper 64 columns), O_k after
    constexpr uint32_t TM_P = kUmmaKeys / 2, TM_O = kUmmaQTiles * kUmmaKeys;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t dyn_smem[];
    // 0 q_full, 1-2 k_full, 3-4 k_empty, 5-6 v_full, 7-8 v_empty,
    // 9-10 s_full[k], 11-12 p_full[k], 13 o_done, 14 drain, 15 q_empty
    __shared__ __align__(8) uint64_t bar[16];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_order[kRankMax];  // sequence of each rank, longest context first
    uint64_t *q_full = &bar[0], *k_full = &bar[1], *k_empty = &bar[3], *v_full = &bar[5],
             *v_empty = &bar[7], *s_full = &bar[9], *p_full = &bar[11], *o_done = &bar[13],
             *drain = &bar[14], *q_empty = &bar[15];
    uint8_t *sq = align_smem_1024(dyn_smem);
    uint8_t *sk = sq + kUmmaQTiles * QB;
    uint8_t *sv = sk + 2 * KVB;

    const int G = a.num_q_heads / a.num_kv_heads;
    const int TT = kUmmaRows / G, rows_used = TT * G;  // query tokens / rows per query tile
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total = a.num_seqs * a.tiles_per_seq * a.num_kv_heads;
    pdl_launch_dependents();
    pdl_wait_prior();
    if (warp == 8 && lane == 0) {
        for (int i = 0; i < 16; ++i) mbar_init(&bar[i], (i == 11 || i == 12) ? 4 : 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (a.num_seqs <= kRankMax) {  // rank of each sequence by context length, ties by index
        int *s_len = reinterpret_cast<int *>(sk);  // the K ring is not in use yet
        for (int i = tid; i < a.num_seqs; i += kUmmaThreads) s_len[i] = a.context_lens[i];
        __syncthreads();
        for (int i = tid; i < a.num_seqs; i += kUmmaThreads) {
            const int key = s_len[i];
            int rk = 0;
            for (int j = 0; j < a.num_seqs; ++j) rk += s_len[j] > key || (s_len[j] == key && j < i);
            s_order[rk] = i;
        }
        fence_proxy_async_smem();  // the K ring held s_len; TMA writes it next
    }
    if (warp == 8) {
        tmem_alloc(&s_tmem, kUmmaTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort_flag = &s_abort;
    // Each role runs to the end of the kernel: the register split of its
    // warpgroup holds until exit, and the teardown is repeated per branch.
    if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == 8 || warp == 10) {
        // ------------------------------------------------------------ producers
        // warp 8 loads each item's query tiles and fills the K ring, warp 10
        // the V ring.  A key tile is 8 blocks x NCH boxes of 16 rows x 128
        // bytes; lane l issues box l (block l / NCH, chunk l % NCH), so the
        // TMA unit sees the tile's boxes from parallel lanes.  Block ids are
        // read from the table in global memory, before the wait for a free
        // stage, so their latency overlaps it.
        const bool is_k = warp == 8;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        uint64_t *full = is_k ? k_full : v_full;
        uint64_t *empty = is_k ? k_empty : v_empty;
        uint8_t *ring = is_k ? sk : sv;
        constexpr int BOXES = 8 * NCH;
        const int bi = lane / NCH, bc = lane % NCH;
        bool ok = true;
        int gt = 0, items = 0;  // key tiles of the items before this one; items started
        int issued = 0;         // key tiles issued
        for (int r = 0; ok; ++r) {
            const int i = umma_round_item(r);
            if (i >= total) break;
            UmmaItem it;
            if (!umma_item(a, s_order, i, G, rows_used, is_k && lane == 0, it)) continue;
            if (is_k) {
                bool freed = true;
                if (lane == 0) {
                    if (items > 0) freed = wait_or_abort(q_empty, (items - 1) & 1, abort_flag);
                    if (freed) {
                        mbar_arrive_expect_tx(q_full, (uint32_t)(kUmmaQTiles * NCH * rows_used * 128));
#pragma unroll
                        for (int k = 0; k < kUmmaQTiles; ++k)
#pragma unroll
                            for (int c = 0; c < NCH; ++c)
                                tma_load_4d(sq + k * QB + c * kUmmaChunk, &tmq, q_full, c * 64, 0,
                                            it.kvh, it.q0 + (it.tile * kUmmaQTiles + k) * TT);
                    }
                }
                ok = __shfl_sync(FULL, freed, 0);
                if (!ok) break;
            }
            ++items;
            for (int j = 0; j < it.ntiles; ++j) {
                const int g = gt + j, st = g & 1;
                const uint32_t ph = (g >> 1) & 1;
                const int blk = j * 8 + bi;
                int id = -1;
                if (lane < BOXES && blk < it.nblk) {
                    id = it.trow[blk];
                    if (id < 0 || id >= a.num_blocks) {
                        flag_error(PA_DEVERR_BLOCK_ID);
                        id = -1;
                    }
                }
                const uint32_t nbox = __popc(__ballot_sync(FULL, id >= 0));
                if (g >= 2) {
                    bool freed = true;
                    if (lane == 0) freed = wait_or_abort(&empty[st], ph ^ 1, abort_flag);
                    ok = __shfl_sync(FULL, freed, 0);
                    if (!ok) break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&full[st], nbox * (uint32_t)(kBlock * 128));
                __syncwarp();
                if (id >= 0)
                    tma_load_2d(ring + st * KVB + bc * kUmmaChunk + bi * 2048, map, &full[st], bc * 64,
                                (id * a.num_kv_heads + it.kvh) * kBlock);
                issued = g + 1;
            }
            gt += it.ntiles;
        }
        if (!ok && lane == 0) {  // let the copies already issued land before the CTA exits
            if (is_k && items > 0) mbar_wait_bounded(q_full, (items - 1) & 1, kWaitTimeoutNs);
            for (int g = max(0, issued - 2); g < issued; ++g)
                mbar_wait_bounded(&full[g & 1], (g >> 1) & 1, kWaitTimeoutNs);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = umma_idesc_f16(FMT, kUmmaRows, kUmmaKeys, 0);
            const uint32_t idesc_pv = umma_idesc_f16(FMT, kUmmaRows, D, 1);
            const uint32_t q_addr = smem_addr(sq), k_addr = smem_addr(sk), v_addr = smem_addr(sv);
            bool issued = false;
            // S_k = Q_k K_g^T, both K-major: a 16-element step is 32 bytes
            // along the swizzled row, the next 64 columns one chunk on
            auto qk = [&](int k, int g) {
                const uint32_t qb = q_addr + k * QB, kb = k_addr + (g & 1) * KVB;
#pragma unroll
                for (int kk = 0; kk < QK_STEPS; ++kk) {
                    const uint32_t off = (kk >> 2) * kUmmaChunk + (kk & 3) * 32;
                    umma_f16_ss(tmem + k * kUmmaKeys, umma_smem_desc(qb + off, 16, 1024),
                                umma_smem_desc(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[k]);
                issued = true;
            };
            // O_k += P_k V_g: P_k from TMEM (16 keys = 8 columns per step), V
            // MN-major (head dim contiguous), a 16-key step 2 KiB further on;
            // the item's first tile starts O_k afresh
            auto pv = [&](int k, int g, bool first) {
                const uint32_t vb = v_addr + (g & 1) * KVB;
#pragma unroll
                for (int kk = 0; kk < PV_STEPS; ++kk)
                    umma_f16_ts(tmem + TM_O + k * D, tmem + k * kUmmaKeys + TM_P + kk * 8,
                                umma_smem_desc(vb + kk * 2048, kUmmaChunk, 1024), idesc_pv,
                                (!first || kk > 0) ? 1u : 0u);
            };
            bool ok = true;
            int gt = 0, items = 0;
            for (int r = 0; ok; ++r) {
                const int i = umma_round_item(r);
                if (i >= total) break;
                UmmaItem it;
                if (!umma_item(a, s_order, i, G, rows_used, false, it)) continue;
                if (!(ok = wait_or_abort(q_full, items & 1, abort_flag) &&
                           wait_or_abort(&k_full[gt & 1], (gt >> 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                qk(0, gt);
                qk(1, gt);
                umma_commit(&k_empty[gt & 1]);
                if (it.ntiles == 1) umma_commit(q_empty);  // the item's last read of Q
                for (int j = 0; j < it.ntiles; ++j) {
                    const int g = gt + j, b = g & 1;
                    const uint32_t ph = (g >> 1) & 1;
                    const bool next = j + 1 < it.ntiles;
                    if (!(ok = wait_or_abort(&v_full[b], ph, abort_flag))) break;
                    if (!(ok = wait_or_abort(&p_full[0], g & 1, abort_flag))) break;
                    tc_fence_after();
                    pv(0, g, j == 0);
                    if (next) {
                        if (!(ok = wait_or_abort(&k_full[b ^ 1], ((g + 1) >> 1) & 1, abort_flag))) break;
                        tc_fence_after();
                        qk(0, g + 1);
                    }
                    if (!(ok = wait_or_abort(&p_full[1], g & 1, abort_flag))) break;
                    tc_fence_after();
                    pv(1, g, j == 0);
                    umma_commit(&v_empty[b]);
                    if (next) {
                        qk(1, g + 1);
                        umma_commit(&k_empty[b ^ 1]);
                        if (j + 2 == it.ntiles) umma_commit(q_empty);
                    }
                }
                if (!ok) break;
                umma_commit(o_done);
                gt += it.ntiles;
                ++items;
            }
            if (issued) {  // the tensor memory stays allocated until every MMA is done
                umma_commit(drain);
                mbar_wait_bounded(drain, 0, kWaitTimeoutNs);
            }
        }
        __syncwarp();
    }
    // every role is done with the tensor memory (loads waited, MMAs complete)
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, kUmmaTmemCols);
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ------------------------------------------------------------ softmax
        const int k = warp >> 2;  // query tile of this warpgroup
        const int r = tid & 127;  // tile row = TMEM lane
        const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t t_s = t_lane + k * kUmmaKeys, t_o = t_lane + TM_O + k * D;
        const float sl2 = a.scale_log2;  // > 0 (checked on the host)
        bool dead = false;
        int gt = 0, items = 0;
        for (int rr = 0; !dead; ++rr) {
            const int i = umma_round_item(rr);
            if (i >= total) break;
            UmmaItem it;
            if (!umma_item(a, s_order, i, G, rows_used, false, it)) continue;
            const int R = it.row0 + k * rows_used + r;
            const bool rvalid = r < rows_used && R < it.rows_total;
            const int qi = rvalid ? R / G : 0, qh = rvalid ? R % G : 0;
            const int pos = rvalid ? it.L - it.n + qi : it.nkeys - 1;  // last key this row sees
            const int live_end = min(it.L, it.nblk * kBlock);  // keys from here on hold no data
            float m_run = kMaskedLogit, l = 0.f;
            for (int j = 0; j < it.ntiles; ++j) {
                const int g = gt + j;
                // blocks of the tile whose id is out of range (read before the wait)
                uint32_t bad = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int blk = j * 8 + q;
                    if (blk < it.nblk) {
                        const int id = it.trow[blk];
                        if (id < 0 || id >= a.num_blocks) bad |= 1u << q;
                    }
                }
                bool ok = wait_or_abort(&s_full[k], g & 1, abort_flag);
                if (!__all_sync(FULL, ok)) {
                    dead = true;
                    break;
                }
                tc_fence_after();
                uint32_t x[kUmmaKeys];
                tmem_ld128(t_s, x);

                const int key0 = j * kUmmaKeys;
                // the max of the raw scores (scale > 0 keeps the order); three-input
                // max, four independent chains
                float mx4[4] = {kMaskedLogit, kMaskedLogit, kMaskedLogit, kMaskedLogit};
                if (key0 + kUmmaKeys - 1 > pos || bad) {
#pragma unroll
                    for (int c = 0; c < kUmmaKeys; ++c) {
                        const bool masked = key0 + c > pos || ((bad >> (c >> 4)) & 1u);
                        if (masked) x[c] = __float_as_uint(kMaskedLogit);
                    }
                }
#pragma unroll
                for (int c = 0; c < kUmmaKeys; c += 2)
                    mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (mx > m_run + kMaxSlack) {
                    alpha = fast_exp2(m_run - mx);
                    m_run = mx;
                    rescale = j > 0;
                }
                // P = 2^(s * scale_log2 - m), 16-bit, two keys per TMEM column,
                // over the upper half of S_k (already read)
                // (one pair in kExp2FmaEvery takes the FMA-pipe 2^a, the rest the
                // special-function unit; scaling and sums run on f32 pairs)
                const uint64_t scale2 = f32x2_pack(sl2, sl2), negm2 = f32x2_pack(-m_run, -m_run);
                uint64_t sum2[2] = {f32x2_pack(0.f, 0.f), f32x2_pack(0.f, 0.f)};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        float a0, a1, p0, p1;
                        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(x[32 * h + 2 * c]),
                                                          __uint_as_float(x[32 * h + 2 * c + 1])),
                                               scale2, negm2),
                                     a0, a1);
                        if (kExp2FmaEvery > 0 && c % kExp2Period == kExp2Period - 1) {
                            exp2_fma_pair(a0, a1, p0, p1);
                        } else {
                            p0 = fast_exp2(a0);
                            p1 = fast_exp2(a1);
                        }
                        sum2[c & 1] = f32x2_add(sum2[c & 1], f32x2_pack(p0, p1));
                        pk[c] = Mma<T>::pack(p0, p1);
                    }
                    tmem_st16(t_s + TM_P + 16 * h, pk);
                }
                float s0, s1, s2, s3;
                f32x2_unpack(sum2[0], s0, s1);
                f32x2_unpack(sum2[1], s2, s3);
                l = l * alpha + ((s0 + s1) + (s2 + s3));
                if (__any_sync(FULL, rescale)) {  // O_k is settled: S_k(g) is complete
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(t_o + c0, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(t_o + c0, o);
                    }
                }
                if (k == 0 && (key0 + kUmmaKeys > live_end || bad)) {
                    // V rows without data (past the context, never loaded, bad
                    // block) meet P = 0 in the MMA; zero them so that whatever
                    // they hold cannot turn 0 * x into NaN
                    ok = wait_or_abort(&v_full[g & 1], (g >> 1) & 1, abort_flag);
                    if (!__all_sync(FULL, ok)) {
                        dead = true;
                        break;
                    }
                    const int key = key0 + r;
                    if (key >= live_end || ((bad >> (r >> 4)) & 1u)) {
                        uint8_t *vrow = sv + (g & 1) * KVB + r * 128;
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                *reinterpret_cast<uint4 *>(vrow + c * kUmmaChunk + u * 16) =
                                    make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[k]);
            }
            if (dead) break;
            // epilogue: O_k / l to the output rows; the item's O_k is complete
            // when o_done's phase for this item has passed
            const bool ok = wait_or_abort(o_done, items & 1, abort_flag);
            if (!__all_sync(FULL, ok)) {
                dead = true;
                break;
            }
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
            uint16_t *orow = reinterpret_cast<uint16_t *>(a.out) +
                             ((size_t)(it.q0 + qi) * a.num_q_heads + (size_t)it.kvh * G + qh) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 64) {
                uint32_t o[64];
                tmem_ld64(t_o + c0, o);
                if (rvalid && out32) {
                    // 32-byte stores: a warp's store covers whole sectors of its
                    // 32 rows, half as many memory transactions as 16-byte ones
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[e] = Mma<T>::pack(__uint_as_float(o[16 * u + 2 * e]) * inv,
                                                __uint_as_float(o[16 * u + 2 * e + 1]) * inv);
                        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(orow + c0 + 16 * u),
                                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                                     : "memory");
                    }
                } else if (rvalid) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        uint4 v;
                        v.x = Mma<T>::pack(__uint_as_float(o[8 * u]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
                        v.y = Mma<T>::pack(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
                        v.z = Mma<T>::pack(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
                        v.w = Mma<T>::pack(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c0 + 8 * u) = v;
                    }
                }
            }
            // the next item's first P.V overwrites O_k: this warp's reads of it
            // are complete (tcgen05.ld waited) before its next arrive
            tc_fence_before();
            gt += it.ntiles;
            ++items;
        }
        tc_fence_before();
        __syncthreads();  // pairs with the teardown barrier of the other warpgroup
    }
}

}  // namespace pa
