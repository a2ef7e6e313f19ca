// Kernels of the paged KV-cache hot path for B200 (sm_100a).
//
//  * scatter_kernel      - pa_reshape_and_cache: one thread per 16-byte
//                          vector of a new token's K and V rows.
//  * copy_blocks_kernel  - pa_copy_blocks: 16-byte vector copy of whole
//                          blocks (all kv heads, K and V).
//  * decode_mma_kernel   - pa_decode with 1..16 query heads per kv head: the
//                          query group is one mma.sync tile against each
//                          16-token K / V tile (the default for every group).
//  * decode_simt_kernel  - pa_decode with one query head per kv head on f32
//                          CUDA cores (selected when built with
//                          PA_MHA_ON_MMA=0).
//  * merge_kernel        - log-sum-exp merge of the partitions of contexts
//                          longer than one partition.
//
// Decode grid: x = sequence * Hkv + kv head, y = partition (slowest, so the
// CTAs of partitions past a short sequence's end, which exit at once, come
// last and overlap the tail of the grid).  A partition covers
// PA_PARTITION_TOKENS tokens (32 blocks), or twice that for calls whose block
// tables span 16384 tokens or more (a.part_blocks).  Inside a CTA each warp owns every
// NW-th block of the partition and runs its own STAGES-deep TMA pipeline:
// one lane loads the warp's next (block, kv head) K and V tiles with
// cp.async.bulk.tensor into a 128-byte-swizzled shared-memory stage and an
// mbarrier tracks the bytes; the warp folds each 16-token tile into a
// running (max, sum, accumulator) online softmax in fp32, log2 domain.  At
// the end the CTA combines its warps; a single-partition sequence writes
// `out`, a split one writes (o, max, sum) to the workspace for merge_kernel.
//
// The kernels are chained with programmatic dependent launch: each kernel
// lets the next one in the stream be scheduled early
// (griddepcontrol.launch_dependents) and waits for the previous one to
// complete before touching global memory (griddepcontrol.wait), which hides
// launch gaps between the scatter, decode and merge kernels.
//
// Tile layout in shared memory (matches the TMA 128-byte swizzle): a 16 x D
// tile is stored as D/64 sub-tiles of 16 rows x 128 bytes; the 16-byte chunk
// c of row r of a sub-tile sits at chunk position c ^ (r & 7).
#pragma once

#include "pa_device.cuh"

#ifndef PA_DECODE_MIN_CTAS
#define PA_DECODE_MIN_CTAS 6  // resident CTAs per SM the <= 8-head decode kernel is compiled for
#endif

namespace pa {

constexpr int kBlock = 16;                                  // tokens per block
constexpr int kPartBlocks = PA_PARTITION_TOKENS / kBlock;   // blocks per partition
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;          // 2 s per wait

struct DecodeArgs {
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;    // [S][Hq][P][D]  normalised partition outputs
    float2 *ws_ml;  // [S][Hq][P]     (max logit in log2 units, sum of 2^(x - max))
    long long num_blocks;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_parts;     // partitions per sequence in the grid
    int part_blocks;   // blocks per partition for this call (the decode kernels
                       // also take it as their PB template argument)
    float scale_log2;  // scale * log2(e)
    // pa_decode_append only (null otherwise): each sequence's new token,
    // [S][Hkv][D], written into the caches at position L - 1 before it is read
    const void *k_new;
    const void *v_new;
    void *key_cache;
    void *value_cache;
};

__device__ __forceinline__ int clamp_context(const DecodeArgs &a, int s, bool report) {
    int L = a.context_lens[s];
    const int cap = a.max_blocks_per_seq * kBlock;
    if (L < 0 || L > cap) {
        if (report) flag_error(PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

// Byte offset of 16-byte chunk `chunk` of row r in a swizzled 16 x D tile.
__device__ __forceinline__ uint32_t tile_off(int r, int chunk) {
    return (uint32_t)((chunk >> 3) * 2048 + r * 128 + (((chunk & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint8_t *align_smem_1024(uint8_t *p) {
    const uint32_t base = smem_addr(p);
    return p + ((1024u - (base & 1023u)) & 1023u);
}

// Sum-reduce 16 per-lane partial dot products across the warp so that lane
// l ends up holding the full sum of value (l >> 1): each xor step keeps the
// half of the values this lane is responsible for and adds the partner's.
__device__ __forceinline__ float reduce16_scatter(float (&v)[16], int lane) {
    const unsigned FULL = 0xffffffffu;
    const bool u4 = lane & 16, u3 = lane & 8, u2 = lane & 4, u1 = lane & 2;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float send = u4 ? v[i] : v[i + 8];
        const float keep = u4 ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = u3 ? v[i] : v[i + 4];
        const float keep = u3 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = u2 ? v[i] : v[i + 2];
        const float keep = u2 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 4);
    }
    {
        const float send = u1 ? v[0] : v[1];
        const float keep = u1 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(FULL, send, 2);
    }
    return v[0] + __shfl_xor_sync(FULL, v[0], 1);
}

// Programmatic dependent launch: let the next kernel in the stream be
// scheduled, and wait until the previous kernel has completed and its memory
// is visible.  Both are no-ops when the launch has no such dependency.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Per-warp TMA pipeline over the warp's blocks of one partition.
template <int D, int STAGES>
struct WarpPipe {
    static constexpr int kTile = kBlock * D * 2;  // bytes of one K (or V) tile
    static constexpr int kStage = 2 * kTile;      // K tile then V tile

    uint8_t *ring;
    uint64_t *bar;
    const CUtensorMap *tmk;
    const CUtensorMap *tmv;
    uint64_t policy;
    int my_phys;  // lane i: physical block of the warp's i-th block, -1 if none/bad
    int kvh, num_kv_heads, lane;

    // Issue the loads of the warp's k-th block into stage k % STAGES.
    // Called by the whole warp; lane 0 issues.
    __device__ __forceinline__ void issue(int k) {
        const int phys = __shfl_sync(0xffffffffu, my_phys, k);
        if (lane == 0) {
            uint64_t *b = &bar[k % STAGES];
            uint8_t *dst = ring + (k % STAGES) * kStage;
            if (phys >= 0) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(b, kStage);
                const int y = (phys * num_kv_heads + kvh) * kBlock;
#pragma unroll
                for (int x = 0; x < D; x += 64) {
                    tma_load_2d_hint(dst + (x / 64) * 2048, tmk, b, x, y, policy);
                    tma_load_2d_hint(dst + kTile + (x / 64) * 2048, tmv, b, x, y, policy);
                }
            } else {
                mbar_arrive(b);  // bad id: the stage completes empty
            }
        }
    }

    // Bounded wait for the k-th block; warp-uniform result.
    __device__ __forceinline__ bool wait(int k) {
        const bool ok = mbar_wait_bounded(&bar[k % STAGES], (k / STAGES) & 1, kWaitTimeoutNs);
        return __all_sync(0xffffffffu, ok);
    }

    // After a failed wait at block k: wait (bounded) for loads still in flight.
    __device__ __forceinline__ void drain(int k, int issued) {
        for (int j = k; j < issued; ++j)
            if (!mbar_wait_bounded(&bar[j % STAGES], (j / STAGES) & 1, kWaitTimeoutNs)) break;
    }
};

__device__ __forceinline__ int warp_block_count(int nb_local, int warp, int nw) {
    return warp < nb_local ? (nb_local - warp + nw - 1) / nw : 0;
}

// pa_decode_append: the warp whose blocks include the one holding position
// L - 1 writes sequence s's new K and V rows for kv head kvh into that slot
// before it issues that block's load.  Each writing lane orders its store
// before the async-proxy (TMA) reads with a proxy fence; the warp then syncs,
// and lane 0 issues the loads.  Other warps and CTAs never read that slot in
// this call (partitions are disjoint token ranges).
//
// append_block_index: the warp's own index k of that block (its k-th block
// is b_begin + warp + k * nw), or -1 when another warp or CTA holds it.  A
// context length that had to be clamped to the table (reported as
// PA_DEVERR_CONTEXT_LEN) writes nothing: position L - 1 is not in the table.
__device__ __forceinline__ int append_block_index(const DecodeArgs &a, int s, int L, int b_begin,
                                                  int nb_local, int warp, int nw) {
    if (a.k_new == nullptr || L <= 0 || a.context_lens[s] != L) return -1;
    const int li = (L - 1) / kBlock - b_begin;
    if (li < 0 || li >= nb_local || li % nw != warp) return -1;
    return li / nw;
}

// The write itself (whole warp).  A bad block id is reported where the block
// is loaded; nothing is written then.
template <int D>
__device__ __forceinline__ void append_new_token(const DecodeArgs &a, int s, int kvh, int L,
                                                 int lane) {
    const int phys = a.block_tables[(size_t)s * a.max_blocks_per_seq + (L - 1) / kBlock];
    if (phys < 0 || phys >= a.num_blocks) return;  // the same for the whole warp
    constexpr int U = D / 8;  // 16-byte units per row: lanes 0..U-1 copy K, U..2U-1 copy V
    if (lane < 2 * U) {
        const bool is_v = lane >= U;
        const int u = is_v ? lane - U : lane;
        const size_t src = ((size_t)s * a.num_kv_heads + kvh) * D + (size_t)u * 8;
        const size_t dst =
            (((size_t)phys * a.num_kv_heads + kvh) * kBlock + (L - 1) % kBlock) * D + (size_t)u * 8;
        const uint4 v =
            *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(is_v ? a.v_new : a.k_new) + src);
        *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(is_v ? a.value_cache : a.key_cache) + dst) = v;
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncwarp();
}

// ------------------------------------------------------------------ decode: one q head per kv head
template <typename T, int D, int NW, int STAGES, int PB>
__global__ void __launch_bounds__(NW * 32)
    decode_simt_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const DecodeArgs a) {
    using Pipe = WarpPipe<D, STAGES>;
    constexpr int EPL = D / 32;  // elements of the head dim per lane
    static_assert(EPL == 2 || EPL == 4, "head_dim 64 or 128");
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[NW][STAGES];
    __shared__ __align__(16) float s_p[NW][kBlock];
    __shared__ __align__(16) float s_acc[NW][D];
    __shared__ float s_m[NW], s_l[NW];

    const int part = blockIdx.y, kvh = blockIdx.x % a.num_kv_heads,
              s = blockIdx.x / a.num_kv_heads;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    pdl_wait_prior();
    const int L = clamp_context(a, s, part == 0 && kvh == 0 && threadIdx.x == 0);
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + PB - 1) / PB;
    if (part >= (nparts > 0 ? nparts : 1)) return;
    const size_t row = (size_t)s * a.num_q_heads + kvh;  // q head == kv head
    uint16_t *out = reinterpret_cast<uint16_t *>(a.out) + row * D;
    if (nblk == 0) {
        for (int i = threadIdx.x; i < D; i += NW * 32) out[i] = 0;
        return;
    }
    const int b_begin = part * PB;
    const int nb_local = min(PB, nblk - b_begin);
    const int nk = warp_block_count(nb_local, warp, NW);

    Pipe pipe;
    pipe.ring = align_smem_1024(dyn_smem) + warp * STAGES * Pipe::kStage;
    pipe.bar = bars[warp];
    pipe.tmk = &tmk;
    pipe.tmv = &tmv;
    pipe.policy = l2_policy_evict_first();
    pipe.kvh = kvh;
    pipe.num_kv_heads = a.num_kv_heads;
    pipe.lane = lane;
    pipe.my_phys = -1;
    if (lane < nk) {
        const int phys =
            a.block_tables[(size_t)s * a.max_blocks_per_seq + b_begin + warp + lane * NW];
        if (phys < 0 || phys >= a.num_blocks)
            flag_error(PA_DEVERR_BLOCK_ID);
        else
            pipe.my_phys = phys;
    }
    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&bars[warp][i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    int issued = nk < STAGES ? nk : STAGES;
    // pa_decode_append: write the new token before the load of its block; if
    // that load is not among the first ones, after them, so that the write's
    // latency overlaps theirs
    const int k_app = append_block_index(a, s, L, b_begin, nb_local, warp, NW);
    if (k_app >= 0 && k_app < issued) append_new_token<D>(a, s, kvh, L, lane);
    for (int k = 0; k < issued; ++k) pipe.issue(k);
    if (k_app >= issued) append_new_token<D>(a, s, kvh, L, lane);

    float qv[EPL];
    {
        const uint16_t *qp = reinterpret_cast<const uint16_t *>(a.q) + row * D + lane * EPL;
        if constexpr (EPL == 4) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(qp);
            const float2 lo = widen2(raw.x, T()), hi = widen2(raw.y, T());
            qv[0] = lo.x; qv[1] = lo.y; qv[2] = hi.x; qv[3] = hi.y;
        } else {
            const float2 f = widen2(*reinterpret_cast<const uint32_t *>(qp), T());
            qv[0] = f.x; qv[1] = f.y;
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) qv[i] *= a.scale_log2;
    }

    float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
    // this lane's 4-byte (EPL 2) or 8-byte (EPL 4) piece of a row: chunk and byte within it
    const int my_chunk = (lane * EPL) / 8;
    const int my_byte = ((lane * EPL) % 8) * 2;

    bool dead = false;
    int k = 0;
    for (; k < nk; ++k) {
        if (!pipe.wait(k)) {
            dead = true;
            break;
        }
        const int phys = __shfl_sync(0xffffffffu, pipe.my_phys, k);
        const int blk = b_begin + warp + k * NW;
        const int nvalid = phys >= 0 ? min(kBlock, L - blk * kBlock) : 0;
        if (nvalid > 0) {
            const uint8_t *kt = pipe.ring + (k % STAGES) * Pipe::kStage;
            const uint8_t *vt = kt + Pipe::kTile;
            float sc[kBlock];
#pragma unroll
            for (int t = 0; t < kBlock; ++t) {
                const uint8_t *src = kt + tile_off(t, my_chunk) + my_byte;
                if constexpr (EPL == 4) {
                    const uint2 raw = *reinterpret_cast<const uint2 *>(src);
                    const float2 lo = widen2(raw.x, T()), hi = widen2(raw.y, T());
                    sc[t] = qv[0] * lo.x + qv[1] * lo.y + qv[2] * hi.x + qv[3] * hi.y;
                } else {
                    const float2 f = widen2(*reinterpret_cast<const uint32_t *>(src), T());
                    sc[t] = qv[0] * f.x + qv[1] * f.y;
                }
            }
            const int tok = lane >> 1;
            float x = reduce16_scatter(sc, lane);
            x = tok < nvalid ? x : -INFINITY;
            float bm = x;
#pragma unroll
            for (int o = 2; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float m_new = fmaxf(m, bm);
            const float alpha = fast_exp2(m - m_new);
            const float p = fast_exp2(x - m_new);
            float ps = p;
#pragma unroll
            for (int o = 2; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l = l * alpha + ps;
            m = m_new;
#pragma unroll
            for (int i = 0; i < EPL; ++i) acc[i] *= alpha;
            if ((lane & 1) == 0) s_p[warp][tok] = p;
            __syncwarp();
            float pv[kBlock];
#pragma unroll
            for (int i = 0; i < kBlock / 4; ++i) {
                const float4 f = reinterpret_cast<const float4 *>(s_p[warp])[i];
                pv[4 * i] = f.x; pv[4 * i + 1] = f.y; pv[4 * i + 2] = f.z; pv[4 * i + 3] = f.w;
            }
#pragma unroll
            for (int t = 0; t < kBlock; ++t) {
                if (t < nvalid) {
                    const uint8_t *src = vt + tile_off(t, my_chunk) + my_byte;
                    if constexpr (EPL == 4) {
                        const uint2 raw = *reinterpret_cast<const uint2 *>(src);
                        const float2 lo = widen2(raw.x, T()), hi = widen2(raw.y, T());
                        acc[0] += pv[t] * lo.x; acc[1] += pv[t] * lo.y;
                        acc[2] += pv[t] * hi.x; acc[3] += pv[t] * hi.y;
                    } else {
                        const float2 f = widen2(*reinterpret_cast<const uint32_t *>(src), T());
                        acc[0] += pv[t] * f.x; acc[1] += pv[t] * f.y;
                    }
                }
            }
        }
        __syncwarp();
        if (issued < nk) pipe.issue(issued++);
    }
    if (dead) {
        pipe.drain(k, issued);
        m = -INFINITY;
        l = 0.f;
    }

#pragma unroll
    for (int i = 0; i < EPL; ++i) s_acc[warp][lane * EPL + i] = acc[i];
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
    __syncthreads();

    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
        if (s_l[w] > 0.f) M = fmaxf(M, s_m[w]);
    float wgt[NW], den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        wgt[w] = s_l[w] > 0.f ? fast_exp2(s_m[w] - M) : 0.f;
        den += wgt[w] * s_l[w];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int i = threadIdx.x; i < D; i += NW * 32) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            if (wgt[w] != 0.f) o += wgt[w] * s_acc[w][i];
        o *= inv;
        if (nparts == 1) {
            out[i] = narrow1(o, T());
        } else {
            a.ws_o[(row * a.num_parts + part) * D + i] = o;
        }
    }
    if (nparts > 1 && threadIdx.x == 0)
        a.ws_ml[row * a.num_parts + part] = make_float2(den > 0.f ? M : -INFINITY, den);
}

// ------------------------------------------------------------------ decode: query group on mma.sync
// NT = number of 8-head column tiles (G <= 8 * NT).  With NT == 1 the kernel
// is compiled for PA_DECODE_MIN_CTAS resident CTAs per SM (80 registers at
// 6): resident warps, not pipeline depth, set the bandwidth this kernel
// reaches.  The 16-head variant holds twice the accumulators; it is
// compiled for 3 CTAs per SM (at most 168 registers), which it reaches
// without spilling.
template <typename T, int D, int NW, int STAGES, int NT, int PB>
__global__ void __launch_bounds__(NW * 32, NT == 1 ? PA_DECODE_MIN_CTAS : 3)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DecodeArgs a) {
    using Pipe = WarpPipe<D, STAGES>;
    constexpr int KS = D / 16;     // 16-wide steps of the head dim
    constexpr int GMAX = 8 * NT;   // query heads per kv head this build handles
    static_assert(GMAX * D * 4 <= STAGES * Pipe::kStage, "combine scratch fits in a warp ring");
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[NW][STAGES];
    __shared__ float s_m[NW][GMAX], s_l[NW][GMAX];

    const int part = blockIdx.y, kvh = blockIdx.x % a.num_kv_heads,
              s = blockIdx.x / a.num_kv_heads;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.num_q_heads / a.num_kv_heads;
    pdl_launch_dependents();
    pdl_wait_prior();
    const int L = clamp_context(a, s, part == 0 && kvh == 0 && threadIdx.x == 0);
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + PB - 1) / PB;
    if (part >= (nparts > 0 ? nparts : 1)) return;
    const size_t row0 = (size_t)s * a.num_q_heads + (size_t)kvh * G;  // first q head of the group
    uint16_t *out = reinterpret_cast<uint16_t *>(a.out) + row0 * D;
    if (nblk == 0) {
        for (int i = threadIdx.x; i < G * D; i += NW * 32) out[i] = 0;
        return;
    }
    const int b_begin = part * PB;
    const int nb_local = min(PB, nblk - b_begin);
    const int nk = warp_block_count(nb_local, warp, NW);

    Pipe pipe;
    pipe.ring = align_smem_1024(dyn_smem) + warp * STAGES * Pipe::kStage;
    pipe.bar = bars[warp];
    pipe.tmk = &tmk;
    pipe.tmv = &tmv;
    pipe.policy = l2_policy_evict_first();
    pipe.kvh = kvh;
    pipe.num_kv_heads = a.num_kv_heads;
    pipe.lane = lane;
    pipe.my_phys = -1;
    if (lane < nk) {
        const int phys =
            a.block_tables[(size_t)s * a.max_blocks_per_seq + b_begin + warp + lane * NW];
        if (phys < 0 || phys >= a.num_blocks)
            flag_error(PA_DEVERR_BLOCK_ID);
        else
            pipe.my_phys = phys;
    }
    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&bars[warp][i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    int issued = nk < STAGES ? nk : STAGES;
    // pa_decode_append: write the new token before the load of its block; if
    // that load is not among the first ones, after them, so that the write's
    // latency overlaps theirs
    const int k_app = append_block_index(a, s, L, b_begin, nb_local, warp, NW);
    if (k_app >= 0 && k_app < issued) append_new_token<D>(a, s, kvh, L, lane);
    for (int k = 0; k < issued; ++k) pipe.issue(k);
    if (k_app >= issued) append_new_token<D>(a, s, kvh, L, lane);

    const int g = lane >> 2, c = lane & 3;
    // B operand of S^T = K Q^T: lane holds Q[h = 8 nt + g][16 kk + 2c .. +1] and [.. + 8 ..].
    uint32_t qf[NT][KS][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + g;
        const uint16_t *qrow = reinterpret_cast<const uint16_t *>(a.q) + (row0 + h) * D;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            qf[nt][kk][0] = h < G ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * c) : 0u;
            qf[nt][kk][1] =
                h < G ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + 2 * c) : 0u;
        }
    }
    // Running softmax state per (tile nt, head 2c + j), and O^T accumulators:
    // acc[nt][j] holds rows d = 16 j + g (+8), columns h = 8 nt + 2c (+1).
    float mrow[NT][2], lrow[NT][2], acc[NT][KS][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        mrow[nt][0] = mrow[nt][1] = -INFINITY;
        lrow[nt][0] = lrow[nt][1] = 0.f;
#pragma unroll
        for (int j = 0; j < KS; ++j) acc[nt][j][0] = acc[nt][j][1] = acc[nt][j][2] = acc[nt][j][3] = 0.f;
    }
    // ldmatrix row/chunk of this lane for the K (A, row-major) and V (A^T) tiles
    const int ka_row = (lane & 7) + ((lane >> 3) & 1) * 8, ka_half = lane >> 4;
    const int va_row = (lane & 7) + 8 * (lane >> 4), va_half = (lane >> 3) & 1;

    bool dead = false;
    int k = 0;
    for (; k < nk; ++k) {
        if (!pipe.wait(k)) {
            dead = true;
            break;
        }
        const int phys = __shfl_sync(0xffffffffu, pipe.my_phys, k);
        const int blk = b_begin + warp + k * NW;
        const int nvalid = phys >= 0 ? min(kBlock, L - blk * kBlock) : 0;
        if (nvalid > 0) {
            uint8_t *kt = pipe.ring + (k % STAGES) * Pipe::kStage;
            uint8_t *vt = kt + Pipe::kTile;
            const uint32_t kt_s = smem_addr(kt), vt_s = smem_addr(vt);
            float sf[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sf[nt][0] = sf[nt][1] = sf[nt][2] = sf[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(af, kt_s + tile_off(ka_row, 2 * kk + ka_half));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) Mma<T>::run(sf[nt], af, qf[nt][kk][0], qf[nt][kk][1]);
            }
            // sf[nt]: (token g, head 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1)
            const bool v0 = g < nvalid, v1 = g + 8 < nvalid;
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float p[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float x0 = v0 ? sf[nt][j] * a.scale_log2 : -INFINITY;
                    const float x1 = v1 ? sf[nt][j + 2] * a.scale_log2 : -INFINITY;
                    float bm = fmaxf(x0, x1);
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
                    const float m_new = fmaxf(mrow[nt][j], bm);
                    const float alpha = fast_exp2(mrow[nt][j] - m_new);
                    p[j] = fast_exp2(x0 - m_new);
                    p[j + 2] = fast_exp2(x1 - m_new);
                    lrow[nt][j] = lrow[nt][j] * alpha + p[j] + p[j + 2];
                    mrow[nt][j] = m_new;
#pragma unroll
                    for (int jj = 0; jj < KS; ++jj) {
                        acc[nt][jj][j] *= alpha;
                        acc[nt][jj][j + 2] *= alpha;
                    }
                }
                // P^T rows g / g+8 (heads 2c, 2c+1) -> B fragments of O^T += V^T P^T
                pb[nt][0] = movmatrix_trans(Mma<T>::pack(p[0], p[1]));
                pb[nt][1] = movmatrix_trans(Mma<T>::pack(p[2], p[3]));
            }
            if (nvalid < kBlock) {
                // rows past the context may hold anything (NaN included): zero them
                for (int idx = lane; idx < (kBlock - nvalid) * (D / 8); idx += 32) {
                    const int t = nvalid + idx / (D / 8), ch = idx % (D / 8);
                    *reinterpret_cast<uint4 *>(vt + tile_off(t, ch)) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < KS; ++j) {
                uint32_t af[4];
                ldmatrix_x4_trans(af, vt_s + tile_off(va_row, 2 * j + va_half));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) Mma<T>::run(acc[nt][j], af, pb[nt][0], pb[nt][1]);
            }
        }
        __syncwarp();
        if (issued < nk) pipe.issue(issued++);
    }
    if (dead) pipe.drain(k, issued);

    // full per-head sums: add the partial sums of the 8 lanes that share c
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float v = lrow[nt][j];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            lrow[nt][j] = dead ? 0.f : v;
        }
    // the warp's ring is idle now: reuse it as [GMAX][D] fp32 scratch
    float *wacc = reinterpret_cast<float *>(pipe.ring);
    if (!dead) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < KS; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = nt * 8 + 2 * c + (e & 1);
                    const int d = 16 * j + g + 8 * (e >> 1);
                    wacc[h * D + d] = acc[nt][j][e];
                }
    }
    if (g == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = nt * 8 + 2 * c + j;
                s_m[warp][h] = mrow[nt][j];
                s_l[warp][h] = lrow[nt][j];
            }
    }
    __syncthreads();

    const uint8_t *rings = align_smem_1024(dyn_smem);
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            if (s_l[w][h] > 0.f) M = fmaxf(M, s_m[w][h]);
        float den = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            if (s_l[w][h] > 0.f) {
                const float wt = fast_exp2(s_m[w][h] - M);
                den += wt * s_l[w][h];
                o += wt * reinterpret_cast<const float *>(rings + w * STAGES * Pipe::kStage)[h * D + d];
            }
        }
        o = den > 0.f ? o / den : 0.f;
        const size_t row = row0 + h;
        if (nparts == 1) {
            out[h * D + d] = narrow1(o, T());
        } else {
            a.ws_o[(row * a.num_parts + part) * D + d] = o;
            if (d == 0) a.ws_ml[row * a.num_parts + part] = make_float2(den > 0.f ? M : -INFINITY, den);
        }
    }
}

// ------------------------------------------------------------------ partition merge
// One warp per (sequence, q head) whose context spans more than one
// partition, kMergeRows rows per CTA: out = sum_p w_p o_p / sum_p w_p with
// w_p = l_p 2^(m_p - M), M = max over partitions that saw a token.  Lane i
// owns partitions i, i + 32, ... for the weights and elements 4i .. 4i + 3 of
// the row (D / 4 lanes) for the sum; weights travel by shuffle, the partial
// rows stream in as independent 16-byte loads.  No block barrier.  A row of
// at most kMergeFew partitions issues all its loads before the reduction.
constexpr int kMergeRows = 4;
constexpr int kMergeFew = 8;  // rows of at most this many partitions load everything at once

template <typename T, int D>
__global__ void __launch_bounds__(kMergeRows * 32) merge_kernel(const DecodeArgs a) {
    pdl_launch_dependents();
    pdl_wait_prior();
    const int lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * kMergeRows + (threadIdx.x >> 5);
    if (row >= (size_t)a.num_seqs * a.num_q_heads) return;
    const int s = (int)(row / a.num_q_heads);
    const int L = clamp_context(a, s, false);
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
    if (nparts <= 1) return;
    const float2 *ml = a.ws_ml + row * a.num_parts;
    constexpr int D4 = D / 4;  // float4 pieces of a row
    const float4 *op = reinterpret_cast<const float4 *>(a.ws_o + row * a.num_parts * D);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (nparts <= kMergeFew) {
        // every load of the row issued at once (the partial rows do not
        // depend on the weights): one round trip to L2 instead of two
        float2 v = lane < nparts ? ml[lane] : make_float2(-INFINITY, 0.f);
        float4 x[kMergeFew];
#pragma unroll
        for (int j = 0; j < kMergeFew; ++j)
            if (j < nparts && lane < D4) x[j] = op[(size_t)j * D4 + lane];
        float M = v.y > 0.f ? v.x : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = v.y > 0.f ? v.y * fast_exp2(v.x - M) : 0.f;
#pragma unroll
        for (int j = 0; j < kMergeFew; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            den += wj;
            if (j < nparts && lane < D4) {
                acc.x += wj * x[j].x; acc.y += wj * x[j].y; acc.z += wj * x[j].z; acc.w += wj * x[j].w;
            }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        if (lane < D4) {
            uint16_t *out = reinterpret_cast<uint16_t *>(a.out) + row * D + 4 * lane;
            const uint32_t lo = (uint32_t)narrow1(acc.x * inv, T()) | ((uint32_t)narrow1(acc.y * inv, T()) << 16);
            const uint32_t hi = (uint32_t)narrow1(acc.z * inv, T()) | ((uint32_t)narrow1(acc.w * inv, T()) << 16);
            *reinterpret_cast<uint2 *>(out) = make_uint2(lo, hi);
        }
        return;
    }
    float M = -INFINITY;
    for (int p = lane; p < nparts; p += 32) {
        const float2 v = ml[p];
        if (v.y > 0.f) M = fmaxf(M, v.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    for (int p0 = 0; p0 < nparts; p0 += 32) {
        const int p = p0 + lane;
        float w = 0.f;
        if (p < nparts) {
            const float2 v = ml[p];
            w = v.y > 0.f ? v.y * fast_exp2(v.x - M) : 0.f;
        }
        den += w;
        const int cnt = min(32, nparts - p0);
#pragma unroll 4
        for (int j = 0; j < cnt; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            if (lane < D4) {
                const float4 x = op[(size_t)(p0 + j) * D4 + lane];
                acc.x += wj * x.x; acc.y += wj * x.y; acc.z += wj * x.z; acc.w += wj * x.w;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (lane < D4) {
        uint16_t *out = reinterpret_cast<uint16_t *>(a.out) + row * D + 4 * lane;
        const uint32_t lo = (uint32_t)narrow1(acc.x * inv, T()) | ((uint32_t)narrow1(acc.y * inv, T()) << 16);
        const uint32_t hi = (uint32_t)narrow1(acc.z * inv, T()) | ((uint32_t)narrow1(acc.w * inv, T()) << 16);
        *reinterpret_cast<uint2 *>(out) = make_uint2(lo, hi);
    }
}

// ------------------------------------------------------------------ scatter write
// grid (token, chunk): each thread moves one 16-byte vector of the token's K
// rows and one of its V rows (vector i = kv head i / (D/8), piece i % (D/8)).
constexpr int kScatterThreads = 128;

template <int D>
__global__ void __launch_bounds__(kScatterThreads)
    scatter_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                   uint4 *__restrict__ kc, uint4 *__restrict__ vc,
                   const int64_t *__restrict__ slots, int num_kv_heads, long long num_slots) {
    constexpr int VPR = D / 8;  // 16-byte vectors per row
    const int t = blockIdx.x;
    const int i = blockIdx.y * kScatterThreads + threadIdx.x;
    pdl_launch_dependents();
    pdl_wait_prior();
    const long long slot = slots[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (blockIdx.y == 0 && threadIdx.x == 0) flag_error(PA_DEVERR_SLOT);
        return;
    }
    if (i >= num_kv_heads * VPR) return;
    const long long b = slot / kBlock, o = slot % kBlock;
    const int h = i / VPR, c = i % VPR;
    const size_t src = (size_t)t * num_kv_heads * VPR + i;
    const size_t dst = (((size_t)b * num_kv_heads + h) * kBlock + o) * VPR + c;
    const uint4 kv = k[src], vv = v[src];
    kc[dst] = kv;
    vc[dst] = vv;
}

// ------------------------------------------------------------------ block copy
// grid.x strides over pairs, grid.y over 16-byte chunks of a block.
__global__ void copy_blocks_kernel(uint4 *__restrict__ kc, uint4 *__restrict__ vc,
                                   const int32_t *__restrict__ pairs, int num_pairs,
                                   long long num_blocks, long long vec_per_block) {
    pdl_launch_dependents();
    pdl_wait_prior();
    for (int p = blockIdx.x; p < num_pairs; p += gridDim.x) {
        const long long src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
            if (blockIdx.y == 0 && threadIdx.x == 0) flag_error(PA_DEVERR_PAIR);
            continue;
        }
        const uint4 *ks = kc + src * vec_per_block;
        const uint4 *vs = vc + src * vec_per_block;
        uint4 *kd = kc + dst * vec_per_block;
        uint4 *vd = vc + dst * vec_per_block;
        for (long long i = (long long)blockIdx.y * blockDim.x + threadIdx.x; i < vec_per_block;
             i += (long long)gridDim.y * blockDim.x) {
            kd[i] = ks[i];
            vd[i] = vs[i];
        }
    }
}

// ------------------------------------------------------------------ chunked prefill
// Multi-query attention of prompt chunks over the paged cache.  Sequence s's
// query rows are the last n_s tokens of its context (their K/V already in
// the cache); token i sits at position L_s - n_s + i and attends to keys
// 0 .. that position.  A CTA takes 64 query rows of one (sequence, kv head):
// row r = token (r / G), group head (r % G); each of its 4 warps owns 16
// rows.  K / V tiles of the sequence's blocks stream through a CTA-wide
// STAGES-deep TMA ring (full barrier: TMA bytes; empty barrier: one arrival
// per warp), and every warp runs the FlashAttention-style inner step on
// mma.sync m16n8k16: S = Q K^T (K through ldmatrix), causal mask and online
// softmax in fp32 (log2 domain), then O += P V with P packed straight from
// the S accumulators and V through ldmatrix.trans.
struct PrefillArgs {
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *query_start;  // [S + 1]
    long long num_blocks;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_q_tokens;
    float scale_log2;
    int tiles_per_seq;  // tcgen05 kernel: CTAs per (sequence, kv head)
};

constexpr float kMaskedLogit = -1.0e30f;  // finite, so 2^(masked - max) is exactly 0

// Shared memory of one prefill CTA beyond its TMA ring: the 64 query rows,
// each padded by 16 bytes so ldmatrix rows fall in different banks.
template <int D>
constexpr int prefill_q_bytes() { return 64 * (D * 2 + 16); }

template <typename T, int D, int STAGES>
__global__ void __launch_bounds__(128, 4)
    prefill_mma_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const PrefillArgs a) {
    constexpr int NW = 4, ROWS = 64, KS = D / 16, NTD = D / 8;
    constexpr int TILE = kBlock * D * 2, STAGE = 2 * TILE;
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    constexpr int QSTRIDE = D * 2 + 16;  // bytes per query row in shared memory
    uint8_t *ring = align_smem_1024(dyn_smem);
    uint8_t *s_q = ring + STAGES * STAGE;
    int32_t *s_table = reinterpret_cast<int32_t *>(s_q + prefill_q_bytes<D>());

    const int G = a.num_q_heads / a.num_kv_heads;
    const int s = blockIdx.x / a.num_kv_heads, kvh = blockIdx.x % a.num_kv_heads;
    const int tile = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    pdl_launch_dependents();
    pdl_wait_prior();
    const int q0 = a.query_start[s];
    int n = a.query_start[s + 1] - q0;
    int L = a.context_lens[s];
    const int cap = a.max_blocks_per_seq * kBlock;
    if (q0 < 0 || q0 > a.num_q_tokens || n > a.num_q_tokens - q0) {  // rows outside q / out
        if (tile == 0 && kvh == 0 && tid == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
        return;
    }
    if (L < 0 || L > cap || n < 0 || n > L) {
        if (tile == 0 && kvh == 0 && tid == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : (L > cap ? cap : L);
        n = n < 0 ? 0 : (n > L ? L : n);
    }
    const int rows_total = n * G;
    if (tile * ROWS >= rows_total) return;
    const int last_row = min(rows_total, (tile + 1) * ROWS) - 1;
    const int nkeys = L - n + last_row / G + 1;  // keys the tile's last row sees
    const int nblk = (nkeys + kBlock - 1) / kBlock;

    // table segment of the blocks this tile reads, checked once
    const int32_t *trow = a.block_tables + (size_t)s * a.max_blocks_per_seq;
    for (int i = tid; i < nblk; i += NW * 32) {
        int b = trow[i];
        if (b < 0 || b >= a.num_blocks) {
            flag_error(PA_DEVERR_BLOCK_ID);
            b = -1;
        }
        s_table[i] = b;
    }
    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], NW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const uint64_t policy = l2_policy_evict_first();
    auto issue = [&](int k) {  // thread 0
        uint64_t *b = &full_bar[k % STAGES];
        uint8_t *dst = ring + (k % STAGES) * STAGE;
        const int phys = s_table[k];
        if (phys >= 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(b, STAGE);
            const int y = (phys * a.num_kv_heads + kvh) * kBlock;
#pragma unroll
            for (int x = 0; x < D; x += 64) {
                tma_load_2d_hint(dst + (x / 64) * 2048, &tmk, b, x, y, policy);
                tma_load_2d_hint(dst + TILE + (x / 64) * 2048, &tmv, b, x, y, policy);
            }
        } else {
            mbar_arrive(b);
        }
    };
    int issued = nblk < STAGES ? nblk : STAGES;
    if (tid == 0)
        for (int k = 0; k < issued; ++k) issue(k);

    // this warp's rows: g and g + 8 of rows tile*64 + warp*16 ..
    const int rbase = tile * ROWS + warp * 16;
    int pos[2];
    bool rvalid[2];
    size_t qrow[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int R = rbase + g + 8 * e;
        rvalid[e] = R < rows_total;
        const int i = rvalid[e] ? R / G : 0, h = rvalid[e] ? R % G : 0;
        pos[e] = rvalid[e] ? L - n + i : -1;
        qrow[e] = ((size_t)(q0 + i) * a.num_q_heads + (size_t)kvh * G + h) * D;
    }
    const int wlast = min(rbase + 15, rows_total - 1);
    const int warp_pmax = wlast >= rbase ? L - n + wlast / G : -1;
    // the CTA's 64 query rows into shared memory (zero rows past the chunk);
    // each warp reads its A fragments from there with ldmatrix per k-step
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q);
        for (int idx = tid; idx < ROWS * (D / 8); idx += NW * 32) {
            const int r = idx / (D / 8), ch = idx % (D / 8);
            const int R = tile * ROWS + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (R < rows_total) {
                const size_t row = (size_t)(q0 + R / G) * a.num_q_heads + (size_t)kvh * G + R % G;
                v = qg[row * (D / 8) + ch];
            }
            *reinterpret_cast<uint4 *>(s_q + r * QSTRIDE + ch * 16) = v;
        }
    }
    __syncthreads();
    const uint32_t q_frag_base =
        smem_addr(s_q) + (uint32_t)((warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * QSTRIDE +
                                    (lane >> 4) * 16);
    float o[NTD][4];
#pragma unroll
    for (int j = 0; j < NTD; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m[2] = {kMaskedLogit, kMaskedLogit}, l[2] = {0.f, 0.f};
    const int k_row = (lane & 7) + 8 * (lane >> 4), k_half = (lane >> 3) & 1;
    const int v_row = (lane & 7) + 8 * ((lane >> 3) & 1), v_half = lane >> 4;

    // Two 16-key blocks per step: the softmax and the rescale check are paid
    // once per 32 keys.
    bool dead = false;
    int k = 0;
    for (; k < nblk; k += 2) {
        const bool two = k + 1 < nblk;
        bool ok = mbar_wait_bounded(&full_bar[k % STAGES], (k / STAGES) & 1, kWaitTimeoutNs);
        if (two)
            ok = mbar_wait_bounded(&full_bar[(k + 1) % STAGES], ((k + 1) / STAGES) & 1,
                                   kWaitTimeoutNs) && ok;
        if (!__all_sync(0xffffffffu, ok)) {
            dead = true;
            break;
        }
        const int key0 = k * kBlock;
        bool use[2];
        use[0] = s_table[k] >= 0 && key0 <= warp_pmax;
        use[1] = two && s_table[k + 1] >= 0 && key0 + kBlock <= warp_pmax;
        if (use[0] || use[1]) {
            uint32_t kt[2], vt[2];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                kt[bb] = smem_addr(ring + ((k + bb) % STAGES) * STAGE);
                vt[bb] = kt[bb] + TILE;
            }
            // sf[2 bb + nt]: block k + bb, keys 8 nt + 2c (+1); rows g / g + 8
            float sf[4][4];
#pragma unroll
            for (int t = 0; t < 4; ++t) sf[t][0] = sf[t][1] = sf[t][2] = sf[t][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t qa[4];
                ldmatrix_x4(qa, q_frag_base + kk * 32);
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    if (!use[bb]) continue;
                    uint32_t b[4];
                    ldmatrix_x4(b, kt[bb] + tile_off(k_row, 2 * kk + k_half));
                    Mma<T>::run(sf[2 * bb], qa, b[0], b[1]);
                    Mma<T>::run(sf[2 * bb + 1], qa, b[2], b[3]);
                }
            }
            float pv[4][4], alpha_row[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {  // row g (e = 0) / g + 8 (e = 1)
                float x[8];
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int key = key0 + 8 * t + 2 * c + u;
                        x[2 * t + u] = (use[t >> 1] && key <= pos[e])
                                           ? sf[t][2 * e + u] * a.scale_log2 : kMaskedLogit;
                    }
                float bm = x[0];
#pragma unroll
                for (int t = 1; t < 8; ++t) bm = fmaxf(bm, x[t]);
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
                const float m_new = fmaxf(m[e], bm);
                const float alpha = fast_exp2(m[e] - m_new);
                float sum = 0.f;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    x[t] = fast_exp2(x[t] - m_new);
                    sum += x[t];
                }
                l[e] = l[e] * alpha + sum;
                m[e] = m_new;
                alpha_row[e] = alpha;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    pv[t][2 * e] = x[2 * t];
                    pv[t][2 * e + 1] = x[2 * t + 1];
                }
            }
            // rescale the accumulators only when some row of the warp raised
            // its running max (alpha < 1); once the max settles this is skipped
            if (__any_sync(0xffffffffu, alpha_row[0] != 1.f || alpha_row[1] != 1.f)) {
#pragma unroll
                for (int j = 0; j < NTD; ++j) {
                    o[j][0] *= alpha_row[0];
                    o[j][1] *= alpha_row[0];
                    o[j][2] *= alpha_row[1];
                    o[j][3] *= alpha_row[1];
                }
            }
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                if (!use[bb]) continue;
                uint32_t pa[4];
                pa[0] = Mma<T>::pack(pv[2 * bb][0], pv[2 * bb][1]);          // row g,     keys 2c..
                pa[1] = Mma<T>::pack(pv[2 * bb][2], pv[2 * bb][3]);          // row g + 8, keys 2c..
                pa[2] = Mma<T>::pack(pv[2 * bb + 1][0], pv[2 * bb + 1][1]);  // row g,     keys 8 + 2c..
                pa[3] = Mma<T>::pack(pv[2 * bb + 1][2], pv[2 * bb + 1][3]);  // row g + 8, keys 8 + 2c..
                // keys past the context (last block) may hold anything: zero
                // their V entries in the fragments
                const int nvalid = min(kBlock, L - (key0 + kBlock * bb));
#pragma unroll
                for (int j = 0; j < NTD; j += 2) {
                    uint32_t b[4];
                    ldmatrix_x4_trans(b, vt[bb] + tile_off(v_row, j + v_half));
                    if (nvalid < kBlock) {
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int kb = 8 * (r & 1) + 2 * c;
                            if (kb >= nvalid) b[r] &= 0xffff0000u;
                            if (kb + 1 >= nvalid) b[r] &= 0x0000ffffu;
                        }
                    }
                    Mma<T>::run(o[j], pa, b[0], b[1]);
                    Mma<T>::run(o[j + 1], pa, b[2], b[3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&empty_bar[k % STAGES]);
            if (two) mbar_arrive(&empty_bar[(k + 1) % STAGES]);
        }
        if (warp == 0) {
            // refill the consumed stages once every warp has released them
            for (int kb = k; kb < k + (two ? 2 : 1) && issued < nblk; ++kb) {
                const bool freed =
                    mbar_wait_bounded(&empty_bar[kb % STAGES], (kb / STAGES) & 1, kWaitTimeoutNs);
                if (!__all_sync(0xffffffffu, freed)) {
                    dead = true;
                    break;
                }
                if (lane == 0) issue(issued);
                ++issued;
            }
            if (dead) {
                k += two ? 2 : 1;
                break;
            }
        }
    }
    if (dead) {
        // wait (bounded) for loads still in flight before the CTA exits
        for (int j = k; j < issued; ++j)
            if (!mbar_wait_bounded(&full_bar[j % STAGES], (j / STAGES) & 1, kWaitTimeoutNs)) break;
        return;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        l[e] += __shfl_xor_sync(0xffffffffu, l[e], 1);
        l[e] += __shfl_xor_sync(0xffffffffu, l[e], 2);
    }
    uint16_t *ob = reinterpret_cast<uint16_t *>(a.out);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        if (!rvalid[e]) continue;
        const float inv = l[e] > 0.f ? 1.f / l[e] : 0.f;
#pragma unroll
        for (int j = 0; j < NTD; ++j) {
            const uint32_t packed =
                (uint32_t)narrow1(o[j][2 * e] * inv, T()) | ((uint32_t)narrow1(o[j][2 * e + 1] * inv, T()) << 16);
            *reinterpret_cast<uint32_t *>(ob + qrow[e] + 8 * j + 2 * c) = packed;
        }
    }
}

// ------------------------------------------------------------------ block swap
// Whole blocks between two pools, either of which may be mapped page-locked
// host memory reached through its device alias: grid.x strides over pairs,
// grid.y over 16-byte chunks of a block.  Ids were checked on the host.
constexpr int kSwapChunk = 2048;  // pairs per launch, passed by value (16 KiB)
struct SwapPairs {
    int2 p[kSwapChunk];
};

__global__ void swap_blocks_kernel(const uint4 *__restrict__ sk, const uint4 *__restrict__ sv,
                                   uint4 *__restrict__ dk, uint4 *__restrict__ dv,
                                   const __grid_constant__ SwapPairs pairs, int num_pairs,
                                   long long vec_per_block) {
    pdl_launch_dependents();
    pdl_wait_prior();
    for (int p = blockIdx.x; p < num_pairs; p += gridDim.x) {
        const int2 pr = pairs.p[p];
        const uint4 *ks = sk + (long long)pr.x * vec_per_block;
        const uint4 *vs = sv + (long long)pr.x * vec_per_block;
        uint4 *kd = dk + (long long)pr.y * vec_per_block;
        uint4 *vd = dv + (long long)pr.y * vec_per_block;
        for (long long i = (long long)blockIdx.y * blockDim.x + threadIdx.x; i < vec_per_block;
             i += (long long)gridDim.y * blockDim.x) {
            const uint4 a = ks[i], b = vs[i];
            kd[i] = a;
            vd[i] = b;
        }
    }
}

// ------------------------------------------------------------------ bounded-wait self test
// One warp waits on a fresh mbarrier that nothing will ever complete, through
// the same bounded wait every kernel above uses; after timeout_ns it records
// PA_DEVERR_TIMEOUT and returns.
__global__ void wait_selftest_kernel(unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    mbar_wait_bounded(&bar, 0, timeout_ns);
}

}  // namespace pa
