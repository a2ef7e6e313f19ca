// Chunked-prefill attention on the fifth-generation tensor cores (tcgen05).
//
// Same operation as prefill_mma_kernel ("PagedAttention in vLLM: a
// throughput settings guide", the chunked-prefill passage: a sequence's new
// tokens attend causally to its whole paged context), as a Blackwell
// warp-specialised pipeline:
//
//  * one CTA = 128 packed query rows (token i, head h of the kv head's query
//    group -> row i * G + h) of one (sequence, kv head);
//  * warp 4 is the producer: TMA loads the query tile once and then, per tile
//    of 128 keys (8 cache blocks), the K and V tiles into two-stage rings; it
//    also owns the tensor-memory allocation;
//  * warp 5, one thread, issues every tcgen05.mma: S = Q K^T into one of two
//    128-column TMEM buffers, and O += P V into a D-column TMEM accumulator,
//    and signals completion with tcgen05.commit;
//  * warps 0-3 (thread r = row r = TMEM lane r) read S rows from TMEM, apply
//    the causal mask, run the online softmax in the log2 domain, write P as
//    16-bit values into a 128-byte-swizzled shared tile, and rescale O in TMEM
//    when the running max has grown; at the end they normalise O and store it.
//
// The S buffers are double-buffered so the tensor core computes S for tile
// j + 1 while the softmax warps work on tile j.  The running max is only
// raised when a tile's max exceeds it by more than 8 (log2 units): until then
// P <= 2^8, which 16-bit P and f32 sums hold exactly as well, and O and l stay
// consistent because both use the same stale max.
//
// Shared-memory tiles are stacks of 8-row x 128-byte atoms in the TMA
// 128-byte swizzle; a 128-row tile of D columns is D / 64 chunks of 16 KiB.
// Every wait is bounded; a wait that gives up raises the CTA's abort flag, the
// other roles leave their loops, in-flight copies and MMAs are waited for,
// and the tensor memory is released before the CTA exits.
#pragma once

#include "pa_kernels.cuh"
#include "pa_umma.cuh"

namespace pa {

constexpr int kUmmaRows = 128;     // packed query rows per CTA (MMA M)
constexpr int kUmmaKeys = 128;     // keys per tile (MMA N of Q K^T, K of P V)
constexpr int kUmmaThreads = 192;  // 4 softmax warps, producer, MMA issuer
constexpr int kUmmaChunk = 128 * 128;  // bytes: 128 rows x 128-byte swizzled chunk
constexpr uint32_t kUmmaTmemCols = 512;
constexpr float kMaxSlack = 8.f;   // log2 growth of the max tolerated before a rescale

template <int D>
constexpr int prefill_umma_smem_bytes() {
    return kUmmaRows * D * 2 + 4 * kUmmaKeys * D * 2 + kUmmaRows * kUmmaKeys * 2 + 1024;
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
    constexpr int QB = kUmmaRows * D * 2;         // query tile bytes
    constexpr int KVB = kUmmaKeys * D * 2;        // one K or V tile
    constexpr int QK_STEPS = D / 16, PV_STEPS = kUmmaKeys / 16;
    constexpr uint32_t FMT = UmmaFormat<T>::value;
    constexpr uint32_t TM_O = 2 * kUmmaKeys;      // TMEM column of O (after S0, S1)
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t dyn_smem[];
    // 0 q_full, 1-2 k_full, 3-4 k_empty, 5-6 v_full, 7-8 v_empty, 9-10 s_full,
    // 11-12 s_empty, 13 p_full, 14 pv_done, 15 drain
    __shared__ __align__(8) uint64_t bar[16];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    uint64_t *q_full = &bar[0], *k_full = &bar[1], *k_empty = &bar[3], *v_full = &bar[5],
             *v_empty = &bar[7], *s_full = &bar[9], *s_empty = &bar[11], *p_full = &bar[13],
             *pv_done = &bar[14], *drain = &bar[15];
    uint8_t *sq = align_smem_1024(dyn_smem);
    uint8_t *sk = sq + QB;
    uint8_t *sv = sk + 2 * KVB;
    uint8_t *sp = sv + 2 * KVB;

    const int G = a.num_q_heads / a.num_kv_heads;
    const int TT = kUmmaRows / G, rows_used = TT * G;  // query tokens / rows per CTA
    const int s = blockIdx.x / a.num_kv_heads, kvh = blockIdx.x % a.num_kv_heads;
    const int tile = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_launch_dependents();
    pdl_wait_prior();
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
    if (tile * rows_used >= rows_total) return;  // nothing allocated yet
    const int last_row = min(rows_total, (tile + 1) * rows_used) - 1;
    const int nkeys = L - n + last_row / G + 1;  // keys the tile's last row sees
    const int nblk = (nkeys + kBlock - 1) / kBlock;
    const int ntiles = (nkeys + kUmmaKeys - 1) / kUmmaKeys;
    const int32_t *trow = a.block_tables + (size_t)s * a.max_blocks_per_seq;

    if (tid == 0) {
        for (int i = 0; i < 16; ++i) mbar_init(&bar[i], (i >= 11 && i <= 13) ? 4 : 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 4) {
        tmem_alloc(&s_tmem, kUmmaTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort_flag = &s_abort;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            int k_issued = 0, v_issued = 0;
            mbar_arrive_expect_tx(q_full, (uint32_t)(NCH * rows_used * 128));
#pragma unroll
            for (int c = 0; c < NCH; ++c)
                tma_load_4d(sq + c * kUmmaChunk, &tmq, q_full, c * 64, 0, kvh, q0 + tile * TT);
            for (int j = 0; j < ntiles; ++j) {
                const int st = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                int ys[8], nvalid = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int blk = j * 8 + i;
                    int y = -1;
                    if (blk < nblk) {
                        const int id = trow[blk];
                        if (id < 0 || id >= a.num_blocks)
                            flag_error(PA_DEVERR_BLOCK_ID);
                        else
                            y = (id * a.num_kv_heads + kvh) * kBlock;
                    }
                    ys[i] = y;
                    nvalid += y >= 0;
                }
                const uint32_t bytes = (uint32_t)(nvalid * kBlock * D * 2);
                if (j >= 2 && !(ok = wait_or_abort(&k_empty[st], ph ^ 1, abort_flag))) break;
                mbar_arrive_expect_tx(&k_full[st], bytes);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (ys[i] >= 0)
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sk + st * KVB + c * kUmmaChunk + i * 2048, &tmk,
                                        &k_full[st], c * 64, ys[i]);
                k_issued = j + 1;
                if (j >= 2 && !(ok = wait_or_abort(&v_empty[st], ph ^ 1, abort_flag))) break;
                mbar_arrive_expect_tx(&v_full[st], bytes);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (ys[i] >= 0)
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sv + st * KVB + c * kUmmaChunk + i * 2048, &tmv,
                                        &v_full[st], c * 64, ys[i]);
                v_issued = j + 1;
            }
            if (!ok) {  // let the copies already issued land before the CTA exits
                mbar_wait_bounded(q_full, 0, kWaitTimeoutNs);
                for (int j = max(0, k_issued - 2); j < k_issued; ++j)
                    mbar_wait_bounded(&k_full[j & 1], (j >> 1) & 1, kWaitTimeoutNs);
                for (int j = max(0, v_issued - 2); j < v_issued; ++j)
                    mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1, kWaitTimeoutNs);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = umma_idesc_f16(FMT, kUmmaRows, kUmmaKeys, 0);
            const uint32_t idesc_pv = umma_idesc_f16(FMT, kUmmaRows, D, 1);
            const uint32_t q_addr = smem_addr(sq), k_addr = smem_addr(sk);
            const uint32_t v_addr = smem_addr(sv), p_addr = smem_addr(sp);
            bool issued = false;
            // O += P V_t: P K-major (keys contiguous), V MN-major (head dim
            // contiguous); a 16-key step is 2 KiB further into the V tile
            auto pv = [&](int t) -> bool {
                if (!wait_or_abort(p_full, t & 1, abort_flag)) return false;
                if (!wait_or_abort(&v_full[t & 1], (t >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vb = v_addr + (t & 1) * KVB;
#pragma unroll
                for (int kk = 0; kk < PV_STEPS; ++kk) {
                    const uint64_t ad =
                        umma_smem_desc(p_addr + (kk >> 2) * kUmmaChunk + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = umma_smem_desc(vb + kk * 2048, kUmmaChunk, 1024);
                    umma_f16_ss(tmem + TM_O, ad, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(pv_done);
                umma_commit(&v_empty[t & 1]);
                return true;
            };
            bool ok = wait_or_abort(q_full, 0, abort_flag);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int b = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                if (j >= 2 && !(ok = wait_or_abort(&s_empty[b], ph ^ 1, abort_flag))) break;
                if (!(ok = wait_or_abort(&k_full[b], ph, abort_flag))) break;
                tc_fence_after();
                const uint32_t kb = k_addr + b * KVB;
                // S_b = Q K^T, both K-major: a 16-element step is 32 bytes
                // along the swizzled row, the next 64 columns one chunk on
#pragma unroll
                for (int kk = 0; kk < QK_STEPS; ++kk) {
                    const uint32_t off = (kk >> 2) * kUmmaChunk + (kk & 3) * 32;
                    umma_f16_ss(tmem + b * kUmmaKeys, umma_smem_desc(q_addr + off, 16, 1024),
                                umma_smem_desc(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                issued = true;
                umma_commit(&s_full[b]);
                umma_commit(&k_empty[b]);
                if (j >= 1) ok = pv(j - 1);
            }
            if (ok) ok = pv(ntiles - 1);
            if (issued) {  // the tensor memory stays allocated until every MMA is done
                umma_commit(drain);
                mbar_wait_bounded(drain, 0, kWaitTimeoutNs);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int rr = tid;  // tile row = TMEM lane
        const int R = tile * rows_used + rr;
        const bool rvalid = rr < rows_used && R < rows_total;
        const int qi = rvalid ? R / G : 0, qh = rvalid ? R % G : 0;
        const int pos = rvalid ? L - n + qi : nkeys - 1;  // last key this row sees
        const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
        const int live_end = min(L, nblk * kBlock);  // keys past it hold no data
        float m_run = kMaskedLogit, l = 0.f;
        bool dead = false;
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            bool ok = wait_or_abort(&s_full[b], ph, abort_flag);
            if (!__all_sync(FULL, ok)) {
                dead = true;
                break;
            }
            tc_fence_after();
            uint32_t x[kUmmaKeys];
            tmem_ld64(t_row + b * kUmmaKeys, reinterpret_cast<uint32_t(&)[64]>(x[0]));
            tmem_ld64(t_row + b * kUmmaKeys + 64, reinterpret_cast<uint32_t(&)[64]>(x[64]));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[b]);

            const int key0 = j * kUmmaKeys;
            uint32_t bad = 0;  // blocks of the tile whose id is out of range
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int blk = j * 8 + q;
                if (blk < nblk) {
                    const int id = trow[blk];
                    if (id < 0 || id >= a.num_blocks) bad |= 1u << q;
                }
            }
            float mx4[4] = {kMaskedLogit, kMaskedLogit, kMaskedLogit, kMaskedLogit};
            if (key0 + kUmmaKeys - 1 > pos || bad) {
#pragma unroll
                for (int c = 0; c < kUmmaKeys; ++c) {
                    const bool masked = key0 + c > pos || ((bad >> (c >> 4)) & 1u);
                    const float v = masked ? kMaskedLogit : __uint_as_float(x[c]) * a.scale_log2;
                    x[c] = __float_as_uint(v);
                    mx4[c & 3] = fmaxf(mx4[c & 3], v);
                }
            } else {
#pragma unroll
                for (int c = 0; c < kUmmaKeys; ++c) {
                    const float v = __uint_as_float(x[c]) * a.scale_log2;
                    x[c] = __float_as_uint(v);
                    mx4[c & 3] = fmaxf(mx4[c & 3], v);
                }
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_run + kMaxSlack) {
                alpha = fast_exp2(m_run - mx);
                m_run = mx;
                rescale = j > 0;
            }
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[kUmmaKeys / 2];
#pragma unroll
            for (int c = 0; c < kUmmaKeys / 2; ++c) {
                const float p0 = fast_exp2(__uint_as_float(x[2 * c]) - m_run);
                const float p1 = fast_exp2(__uint_as_float(x[2 * c + 1]) - m_run);
                sum4[c & 3] += p0 + p1;
                pk[c] = Mma<T>::pack(p0, p1);
            }
            l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));

            if (j > 0) {  // P V_{j-1} done: the P tile is free and O is settled
                ok = wait_or_abort(pv_done, (j - 1) & 1, abort_flag);
                if (!__all_sync(FULL, ok)) {
                    dead = true;
                    break;
                }
                tc_fence_after();
            }
            if (key0 + kUmmaKeys > live_end || bad) {
                // V rows without data (past the context, never loaded, bad
                // block) would meet P = 0 in the MMA; zero them so that
                // whatever they hold cannot turn 0 * x into NaN
                ok = wait_or_abort(&v_full[b], ph, abort_flag);
                if (!__all_sync(FULL, ok)) {
                    dead = true;
                    break;
                }
                const int key = key0 + rr;
                if (key >= live_end || ((bad >> (rr >> 4)) & 1u)) {
                    uint8_t *vrow = sv + b * KVB + rr * 128;
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<uint4 *>(vrow + c * kUmmaChunk + u * 16) =
                                make_uint4(0, 0, 0, 0);
                }
            }
            if (__any_sync(FULL, rescale)) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 64) {
                    uint32_t o[64];
                    tmem_ld64(t_row + TM_O + c0, o);
#pragma unroll
                    for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st64(t_row + TM_O + c0, o);
                }
                tmem_wait_st();
            }
            // row rr of P: 16-byte chunk u of 128-byte chunk c at u ^ (rr & 7)
            uint8_t *prow = sp + rr * 128;
#pragma unroll
            for (int u = 0; u < 16; ++u)
                *reinterpret_cast<uint4 *>(prow + (u >> 3) * kUmmaChunk + (((u & 7) ^ (rr & 7)) << 4)) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (!dead) {
            const bool ok = wait_or_abort(pv_done, (ntiles - 1) & 1, abort_flag);
            if (__all_sync(FULL, ok)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                uint16_t *orow = reinterpret_cast<uint16_t *>(a.out) +
                                 ((size_t)(q0 + qi) * a.num_q_heads + (size_t)kvh * G + qh) * D;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 64) {
                    uint32_t o[64];
                    tmem_ld64(t_row + TM_O + c0, o);
                    if (rvalid) {
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
    }
    // every role is done with the tensor memory (loads waited, MMAs complete)
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, kUmmaTmemCols);
    }
}

}  // namespace pa
