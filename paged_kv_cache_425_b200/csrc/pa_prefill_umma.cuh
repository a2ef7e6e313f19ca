// Chunked-prefill attention on the fifth-generation tensor cores (tcgen05).
//
// Same operation as prefill_mma_kernel ("PagedAttention in vLLM: a
// throughput settings guide", the chunked-prefill passage: a sequence's new
// tokens attend causally to its whole paged context), as a Blackwell
// warp-specialised pipeline.  One CTA owns two query tiles of 128 packed rows
// (token i, head h of the kv head's query group -> row i * G + h) of one
// (sequence, kv head) and walks the context in tiles of 128 keys (8 blocks):
//
//  * warp 8 is the producer: TMA loads both query tiles once, then each
//    key tile's K and V blocks into two-stage rings; it owns the TMEM
//    allocation;
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
// Warps 10 and 11 only complete the third warpgroup (setmaxnreg works per
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

// Dynamic shared memory: both query tiles, two K and two V stages, the
// CTA's block-table segment, and alignment slack.
template <int D>
constexpr int prefill_umma_smem_bytes(int table_entries) {
    return kUmmaQTiles * kUmmaRows * D * 2 + 4 * kUmmaKeys * D * 2 + 1024 + 4 * table_entries;
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
    // 9-10 s_full[k], 11-12 p_full[k], 13 o_done, 14 drain
    __shared__ __align__(8) uint64_t bar[15];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    uint64_t *q_full = &bar[0], *k_full = &bar[1], *k_empty = &bar[3], *v_full = &bar[5],
             *v_empty = &bar[7], *s_full = &bar[9], *p_full = &bar[11], *o_done = &bar[13],
             *drain = &bar[14];
    uint8_t *sq = align_smem_1024(dyn_smem);
    uint8_t *sk = sq + kUmmaQTiles * QB;
    uint8_t *sv = sk + 2 * KVB;
    int32_t *s_table = reinterpret_cast<int32_t *>(sv + 2 * KVB);

    const int G = a.num_q_heads / a.num_kv_heads;
    const int TT = kUmmaRows / G, rows_used = TT * G;  // query tokens / rows per query tile
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA index -> (sequence rank, query tile from the last, kv head).  The
    // block scheduler hands CTAs to SMs in index order as SMs free up, so
    // numbering the longest contexts first makes it a longest-first list
    // schedule: the short CTAs fill in the tail.
    const int per_seq = a.tiles_per_seq * a.num_kv_heads;
    const int rank = blockIdx.x / per_seq, rem = blockIdx.x % per_seq;
    const int tile = a.tiles_per_seq - 1 - rem / a.num_kv_heads, kvh = rem % a.num_kv_heads;
    __shared__ int s_len[kRankMax];
    __shared__ int s_pick;
    pdl_launch_dependents();
    pdl_wait_prior();
    int s = rank;
    if (a.num_seqs <= kRankMax) {  // sequence of this rank by context length, ties by index
        for (int i = tid; i < a.num_seqs; i += kUmmaThreads) s_len[i] = a.context_lens[i];
        __syncthreads();
        for (int i = tid; i < a.num_seqs; i += kUmmaThreads) {
            const int key = s_len[i];
            int rk = 0;
            for (int j = 0; j < a.num_seqs; ++j) rk += s_len[j] > key || (s_len[j] == key && j < i);
            if (rk == rank) s_pick = i;
        }
        __syncthreads();
        s = s_pick;
    }
    const int q0 = a.query_start[s];
    int n = a.query_start[s + 1] - q0;
    int L = a.context_lens[s];
    const int cap = a.max_blocks_per_seq * kBlock;
    if (q0 < 0 || q0 > a.num_q_tokens || n > a.num_q_tokens - q0) {
        if (tile == 0 && kvh == 0 && tid == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
        return;
    }
    if (L < 0 || L > cap || n < 0 || n > L) {
        if (tile == 0 && kvh == 0 && tid == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : (L > cap ? cap : L);
        n = n < 0 ? 0 : (n > L ? L : n);
    }
    const int rows_total = n * G;
    const int row0 = tile * kUmmaQTiles * rows_used;  // first packed row of the CTA
    if (row0 >= rows_total) return;                   // nothing allocated yet
    const int last_row = min(rows_total, row0 + kUmmaQTiles * rows_used) - 1;
    const int nkeys = L - n + last_row / G + 1;       // keys the CTA's last row sees
    const int nblk = (nkeys + kBlock - 1) / kBlock;
    const int ntiles = (nkeys + kUmmaKeys - 1) / kUmmaKeys;
    const int32_t *trow = a.block_tables + (size_t)s * a.max_blocks_per_seq;

    // The producer thread sets up the barriers and starts the query-tile load
    // before the CTA stages its block ids, so its latency overlaps the setup.
    if (warp == 8 && lane == 0) {
        for (int i = 0; i < 15; ++i) mbar_init(&bar[i], (i == 11 || i == 12) ? 4 : 1);
        fence_mbar_init();
        s_abort = 0;
        mbar_arrive_expect_tx(q_full, (uint32_t)(kUmmaQTiles * NCH * rows_used * 128));
#pragma unroll
        for (int k = 0; k < kUmmaQTiles; ++k)
#pragma unroll
            for (int c = 0; c < NCH; ++c)
                tma_load_4d(sq + k * QB + c * kUmmaChunk, &tmq, q_full, c * 64, 0, kvh,
                            q0 + (tile * kUmmaQTiles + k) * TT);
    }
    // the CTA's block ids, checked once: -1 marks an id out of range
    for (int i = tid; i < nblk; i += kUmmaThreads) {
        int b = trow[i];
        if (b < 0 || b >= a.num_blocks) {
            flag_error(PA_DEVERR_BLOCK_ID);
            b = -1;
        }
        s_table[i] = b;
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
        // warp 8 fills the K ring, warp 10 the V ring.  A key tile is 8 blocks
        // x NCH boxes of 16 rows x 128 bytes; lane l issues box l (block l / NCH,
        // chunk l % NCH), so the TMA unit sees the tile's boxes from parallel
        // lanes, not one thread's serial stream (one issuing thread leaves it
        // well short of the rate the GEMMs consume K and V at).
        const bool is_k = warp == 8;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        uint64_t *full = is_k ? k_full : v_full;
        uint64_t *empty = is_k ? k_empty : v_empty;
        uint8_t *ring = is_k ? sk : sv;
        constexpr int BOXES = 8 * NCH;
        const int bi = lane / NCH, bc = lane % NCH;
        bool ok = true;
        int issued = 0;
        for (int j = 0; j < ntiles; ++j) {
            const int st = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            const int blk = j * 8 + bi;
            const int id = (lane < BOXES && blk < nblk) ? s_table[blk] : -1;
            const uint32_t nbox = __popc(__ballot_sync(FULL, id >= 0));
            if (j >= 2) {
                bool freed = true;
                if (lane == 0) freed = wait_or_abort(&empty[st], ph ^ 1, abort_flag);
                ok = __shfl_sync(FULL, freed, 0);
                if (!ok) break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[st], nbox * (uint32_t)(kBlock * 128));
            __syncwarp();
            if (id >= 0)
                tma_load_2d(ring + st * KVB + bc * kUmmaChunk + bi * 2048, map, &full[st], bc * 64,
                            (id * a.num_kv_heads + kvh) * kBlock);
            issued = j + 1;
        }
        if (!ok && lane == 0) {  // let the copies already issued land before the CTA exits
            if (is_k) mbar_wait_bounded(q_full, 0, kWaitTimeoutNs);
            for (int j = max(0, issued - 2); j < issued; ++j)
                mbar_wait_bounded(&full[j & 1], (j >> 1) & 1, kWaitTimeoutNs);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = umma_idesc_f16(FMT, kUmmaRows, kUmmaKeys, 0);
            const uint32_t idesc_pv = umma_idesc_f16(FMT, kUmmaRows, D, 1);
            const uint32_t q_addr = smem_addr(sq), k_addr = smem_addr(sk), v_addr = smem_addr(sv);
            bool issued = false;
            // S_k = Q_k K_j^T, both K-major: a 16-element step is 32 bytes
            // along the swizzled row, the next 64 columns one chunk on
            auto qk = [&](int k, int j) {
                const uint32_t qb = q_addr + k * QB, kb = k_addr + (j & 1) * KVB;
#pragma unroll
                for (int kk = 0; kk < QK_STEPS; ++kk) {
                    const uint32_t off = (kk >> 2) * kUmmaChunk + (kk & 3) * 32;
                    umma_f16_ss(tmem + k * kUmmaKeys, umma_smem_desc(qb + off, 16, 1024),
                                umma_smem_desc(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[k]);
                issued = true;
            };
            // O_k += P_k V_j: P_k from TMEM (16 keys = 8 columns per step), V
            // MN-major (head dim contiguous), a 16-key step 2 KiB further on
            auto pv = [&](int k, int j) {
                const uint32_t vb = v_addr + (j & 1) * KVB;
#pragma unroll
                for (int kk = 0; kk < PV_STEPS; ++kk)
                    umma_f16_ts(tmem + TM_O + k * D, tmem + k * kUmmaKeys + TM_P + kk * 8,
                                umma_smem_desc(vb + kk * 2048, kUmmaChunk, 1024), idesc_pv,
                                (j > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = wait_or_abort(q_full, 0, abort_flag) &&
                      wait_or_abort(&k_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                qk(1, 0);
                umma_commit(&k_empty[0]);
            }
            for (int j = 0; ok && j < ntiles; ++j) {
                const int b = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                const bool next = j + 1 < ntiles;
                if (!(ok = wait_or_abort(&v_full[b], ph, abort_flag))) break;
                if (!(ok = wait_or_abort(&p_full[0], j & 1, abort_flag))) break;
                tc_fence_after();
                pv(0, j);
                if (next) {
                    if (!(ok = wait_or_abort(&k_full[b ^ 1], ((j + 1) >> 1) & 1, abort_flag))) break;
                    tc_fence_after();
                    qk(0, j + 1);
                }
                if (!(ok = wait_or_abort(&p_full[1], j & 1, abort_flag))) break;
                tc_fence_after();
                pv(1, j);
                umma_commit(&v_empty[b]);
                if (next) {
                    qk(1, j + 1);
                    umma_commit(&k_empty[b ^ 1]);
                }
            }
            if (ok) umma_commit(o_done);
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
        const int R = row0 + k * rows_used + r;
        const bool rvalid = r < rows_used && R < rows_total;
        const int qi = rvalid ? R / G : 0, qh = rvalid ? R % G : 0;
        const int pos = rvalid ? L - n + qi : nkeys - 1;  // last key this row sees
        const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t t_s = t_lane + k * kUmmaKeys, t_o = t_lane + TM_O + k * D;
        const int live_end = min(L, nblk * kBlock);  // keys from here on hold no data
        const float sl2 = a.scale_log2;               // > 0 (checked on the host)
        float m_run = kMaskedLogit, l = 0.f;
        bool dead = false;
        for (int j = 0; j < ntiles; ++j) {
            bool ok = wait_or_abort(&s_full[k], j & 1, abort_flag);
            if (!__all_sync(FULL, ok)) {
                dead = true;
                break;
            }
            tc_fence_after();
            uint32_t x[kUmmaKeys];
            tmem_ld128(t_s, x);

            const int key0 = j * kUmmaKeys;
            uint32_t bad = 0;  // blocks of the tile whose id is out of range
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int blk = j * 8 + q;
                if (blk < nblk && s_table[blk] < 0) bad |= 1u << q;
            }
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
            if (__any_sync(FULL, rescale)) {  // O_k is settled: S_k(j) is complete
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
                ok = wait_or_abort(&v_full[j & 1], (j >> 1) & 1, abort_flag);
                if (!__all_sync(FULL, ok)) {
                    dead = true;
                    break;
                }
                const int key = key0 + r;
                if (key >= live_end || ((bad >> (r >> 4)) & 1u)) {
                    uint8_t *vrow = sv + (j & 1) * KVB + r * 128;
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
        if (!dead) {
            const bool ok = wait_or_abort(o_done, 0, abort_flag);
            if (__all_sync(FULL, ok)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
                uint16_t *orow = reinterpret_cast<uint16_t *>(a.out) +
                                 ((size_t)(q0 + qi) * a.num_q_heads + (size_t)kvh * G + qh) * D;
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
                            for (int i = 0; i < 8; ++i)
                                w[i] = Mma<T>::pack(__uint_as_float(o[16 * u + 2 * i]) * inv,
                                                    __uint_as_float(o[16 * u + 2 * i + 1]) * inv);
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
            }
        }
        tc_fence_before();
        __syncthreads();  // pairs with the teardown barrier of the other warpgroup
    }
}

}  // namespace pa
