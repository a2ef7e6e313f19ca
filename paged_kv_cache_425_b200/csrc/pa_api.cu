// Host side of libpa.so: argument checks, TMA descriptor encoding and kernel
// launches for the entry points declared in include/pa_api.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "pa_api.h"
#include "pa_kernels.cuh"
#include "pa_prefill_umma.cuh"

namespace pa {
namespace {

// Decode launch shape: warps per CTA and TMA stages per warp (build-time
// overridable for tuning sweeps).
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_STAGES_128
#define PA_STAGES_128 1  // 1 x 8 KiB per warp at head_dim 128: 6 CTAs per SM
#endif
#ifndef PA_STAGES_64
#define PA_STAGES_64 2   // 2 x 4 KiB per warp at head_dim 64
#endif
#ifndef PA_MHA_ON_MMA
#define PA_MHA_ON_MMA 1  // 0: one query head per kv head takes the f32 CUDA-core kernel
#endif
constexpr int kWarps = PA_DECODE_WARPS;
constexpr int kStages128 = PA_STAGES_128;
constexpr int kStages64 = PA_STAGES_64;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// TMA descriptor of a cache viewed as 2-D: rows = num_blocks * num_kv_heads *
// 16 (one per token slot), columns = head_dim; box = 16 rows x 64 columns
// (128 bytes), 128-byte swizzle.
bool encode_cache_map(CUtensorMap *map, const void *cache, int64_t num_blocks, int num_kv_heads,
                      int head_dim, int dtype) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)head_dim,
                          (cuuint64_t)num_blocks * (cuuint64_t)num_kv_heads * kBlock};
    cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kBlock};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    2, const_cast<void *>(cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// TMA descriptor of the query rows of one kv head's group, viewed as 4-D:
// (head_dim, G heads of the group, kv head, token), box = 64 columns x G x 1 x
// TT tokens, so a box lands as TT * G rows of 128 bytes in packed-row order
// (token i, head h -> row i * G + h); 128-byte swizzle; rows past the last
// token read as zero.
bool encode_q_map(CUtensorMap *map, const void *q, int num_q_tokens, int num_q_heads,
                  int num_kv_heads, int head_dim, int dtype, int tokens_per_box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int G = num_q_heads / num_kv_heads;
    cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)G, (cuuint64_t)num_kv_heads,
                          (cuuint64_t)num_q_tokens};
    cuuint64_t strides[3] = {(cuuint64_t)head_dim * 2, (cuuint64_t)G * head_dim * 2,
                             (cuuint64_t)num_q_heads * head_dim * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)tokens_per_box};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    4, const_cast<void *>(q), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

std::atomic<int> g_prefill_kernel{PA_PREFILL_AUTO};

int check_cache_shape(int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int64_t num_blocks, int32_t dtype) {
    if (num_kv_heads <= 0 || num_blocks <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (block_size != kBlock) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (num_blocks * (int64_t)num_kv_heads * kBlock >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel in the stream finishes; it waits for that kernel
// (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (ids are never reused
// within a process, unlike context handles), or 0 when there is none yet or
// the driver cannot say.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` (once per kernel,
// device, CUDA context and size: the attribute persists in the context, and a
// device reset starts a new one).
template <typename Kernel>
bool set_smem(Kernel k, int bytes) {
    struct Key {
        const void *fn;
        int dev, bytes;
        unsigned long long ctx;
    };
    static std::mutex mu;
    static std::vector<Key> done;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const unsigned long long ctx = current_context_id();
    const void *fn = reinterpret_cast<const void *>(k);
    std::lock_guard<std::mutex> lock(mu);
    for (const Key &e : done)
        if (ctx != 0 && e.fn == fn && e.dev == dev && e.ctx == ctx && e.bytes >= bytes) return true;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    if (ctx != 0) done.push_back({fn, dev, bytes, ctx});
    return true;
}

// Registers per thread a kernel was compiled with (-1 on failure); looked up
// once per kernel, device and CUDA context.
template <typename Kernel>
int compiled_registers(Kernel k) {
    struct Entry {
        const void *fn;
        int dev, regs;
        unsigned long long ctx;
    };
    static std::mutex mu;
    static std::vector<Entry> seen;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    const unsigned long long ctx = current_context_id();
    const void *fn = reinterpret_cast<const void *>(k);
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &e : seen)
        if (ctx != 0 && e.fn == fn && e.dev == dev && e.ctx == ctx) return e.regs;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return -1;
    if (ctx != 0) seen.push_back({fn, dev, fa.numRegs, ctx});
    return fa.numRegs;
}

// Streaming multiprocessors of the current device (-1 on failure); looked up
// once per device.
int sm_count() {
    static std::mutex mu;
    static std::vector<std::pair<int, int>> seen;  // (device, SMs)
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    for (const auto &e : seen)
        if (e.first == dev) return e.second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    seen.push_back({dev, n});
    return n;
}

template <typename T, int D, int PB>
int launch_decode(const DecodeArgs &a, int group, const CUtensorMap &tmk, const CUtensorMap &tmv,
                  cudaStream_t st) {
    constexpr int STAGES = D == 128 ? kStages128 : kStages64;
    constexpr int SMEM = kWarps * STAGES * WarpPipe<D, STAGES>::kStage + 1024;
    const dim3 grid(a.num_seqs * a.num_kv_heads, a.num_parts);
    const dim3 block(kWarps * 32);
    int rc;
    if (group == 1 && !PA_MHA_ON_MMA) {
        auto k = decode_simt_kernel<T, D, kWarps, STAGES, PB>;
        if (!set_smem(k, SMEM)) return PA_ERR_CUDA;
        rc = launch_pdl(k, grid, block, SMEM, st, tmk, tmv, a);
    } else if (group <= 8) {
        auto k = decode_mma_kernel<T, D, kWarps, STAGES, 1, PB>;
        if (!set_smem(k, SMEM)) return PA_ERR_CUDA;
        rc = launch_pdl(k, grid, block, SMEM, st, tmk, tmv, a);
    } else {
        auto k = decode_mma_kernel<T, D, kWarps, STAGES, 2, PB>;
        if (!set_smem(k, SMEM)) return PA_ERR_CUDA;
        rc = launch_pdl(k, grid, block, SMEM, st, tmk, tmv, a);
    }
    if (rc != PA_OK || a.num_parts <= 1) return rc;
    const int64_t rows = (int64_t)a.num_seqs * a.num_q_heads;
    return launch_pdl(merge_kernel<T, D>, dim3((unsigned)((rows + kMergeRows - 1) / kMergeRows)),
                      dim3(kMergeRows * 32), 0, st, a);
}

template <typename T>
int dispatch_decode(const DecodeArgs &a, int head_dim, int group, const CUtensorMap &tmk,
                    const CUtensorMap &tmv, cudaStream_t st) {
    // the partition length is a compile-time constant of the decode kernels
    // (a runtime value measured ~2.5 % slower on the Llama-7B shape)
    if (a.part_blocks == 2 * kPartBlocks)
        return head_dim == 128 ? launch_decode<T, 128, 2 * kPartBlocks>(a, group, tmk, tmv, st)
                               : launch_decode<T, 64, 2 * kPartBlocks>(a, group, tmk, tmv, st);
    return head_dim == 128 ? launch_decode<T, 128, kPartBlocks>(a, group, tmk, tmv, st)
                           : launch_decode<T, 64, kPartBlocks>(a, group, tmk, tmv, st);
}

// Device-side address of `p` on the current device: itself for device memory
// of this device, the mapped alias for page-locked host memory.  False for
// pageable host memory, another device's memory or a lookup failure.
bool device_alias(const void *p, const void **out) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (attr.type == cudaMemoryTypeDevice && attr.device == dev && attr.devicePointer) {
        *out = p;
        return true;
    }
    if (attr.type == cudaMemoryTypeHost && attr.devicePointer) {
        *out = attr.devicePointer;
        return true;
    }
    return false;
}

// Blocks per decode partition: PA_PARTITION_TOKENS, doubled when the block
// tables span 16384 tokens or more.  Long contexts then split into fewer,
// longer partitions: fewer partials to merge and less per-CTA overhead,
// while short-context batches keep the parallelism of the shorter ones
// (measured: 1024-token partitions +3 % on 8k-32k contexts, -4 % on
// contexts up to 2k).
constexpr int kWideTableTokens = 16384;
int part_blocks_for(int32_t max_blocks_per_seq) {
    return (int64_t)max_blocks_per_seq * kBlock >= kWideTableTokens ? 2 * kPartBlocks : kPartBlocks;
}

int64_t num_parts_for(int32_t max_blocks_per_seq) {
    const int pb = part_blocks_for(max_blocks_per_seq);
    return (max_blocks_per_seq + pb - 1) / pb;
}

// Workspace: partition outputs fp32 [S][Hq][P][D], then (max, sum) float2
// [S][Hq][P]; each region starts on a 256-byte boundary.
struct WorkspaceLayout {
    int64_t o_off, ml_off, total;
};

WorkspaceLayout workspace_layout(int64_t num_seqs, int64_t num_q_heads, int64_t head_dim,
                                 int64_t parts) {
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t rows = num_seqs * num_q_heads * parts;
    WorkspaceLayout l;
    l.o_off = 0;
    l.ml_off = up(rows * head_dim * 4);
    l.total = l.ml_off + up(rows * 8);
    return l;
}

// pa_prefill on the tcgen05 kernel: work items of two query tiles of 128
// packed rows (the largest multiple of the group size <= 128) per (sequence,
// kv head), walked by one persistent CTA per SM.
int launch_prefill_umma(void *out, const void *q, const void *key_cache, const void *value_cache,
                        const int32_t *block_tables, const int32_t *context_lens,
                        const int32_t *query_start, int32_t max_query_len, int32_t num_kv_heads,
                        float scale, int32_t num_seqs, int32_t num_q_heads, int32_t num_q_tokens,
                        int32_t head_dim, int32_t max_blocks_per_seq, int64_t num_blocks,
                        int32_t dtype, cudaStream_t st) {
    const int group = num_q_heads / num_kv_heads;
    const int tokens_per_tile = kUmmaRows / group;
    const int64_t rows_per_cta = (int64_t)kUmmaQTiles * tokens_per_tile * group;
    const int64_t tiles = ((int64_t)max_query_len * group + rows_per_cta - 1) / rows_per_cta;
    PrefillArgs a;
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start = query_start;
    a.num_blocks = num_blocks;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_q_tokens = num_q_tokens;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.tiles_per_seq = (int)tiles;
    CUtensorMap tmq, tmk, tmv;
    if (!encode_q_map(&tmq, q, num_q_tokens, num_q_heads, num_kv_heads, head_dim, dtype,
                      tokens_per_tile) ||
        !encode_cache_map(&tmk, key_cache, num_blocks, num_kv_heads, head_dim, dtype) ||
        !encode_cache_map(&tmv, value_cache, num_blocks, num_kv_heads, head_dim, dtype))
        return PA_ERR_CUDA;
    const int64_t items = (int64_t)num_seqs * num_kv_heads * tiles;
    if (items >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    // persistent: one CTA per SM (tensor memory and shared memory allow no
    // second), each walking its share of the items
    const int sms = sm_count();
    if (sms <= 0) return PA_ERR_CUDA;
    const dim3 grid((unsigned)std::min<int64_t>(items, sms));
    const int smem = head_dim == 128 ? prefill_umma_smem_bytes<128>() : prefill_umma_smem_bytes<64>();
    auto launch = [&](auto kernel) -> int {
        // the kernel re-splits its registers per warpgroup (setmaxnreg); a
        // split above what the launch holds would wait forever, so check the
        // compiled count first
        const int regs = compiled_registers(kernel);
        if (regs < 0) return PA_ERR_CUDA;
        if ((int64_t)regs * kUmmaThreads < kUmmaRegsNeeded) return PA_ERR_UNSUPPORTED;
        if (!set_smem(kernel, smem)) return PA_ERR_CUDA;
        return launch_pdl(kernel, grid, dim3(kUmmaThreads), (size_t)smem, st, tmq, tmk, tmv, a);
    };
    if (dtype == PA_F16)
        return head_dim == 128 ? launch(prefill_umma_kernel<__half, 128>)
                               : launch(prefill_umma_kernel<__half, 64>);
    return head_dim == 128 ? launch(prefill_umma_kernel<__nv_bfloat16, 128>)
                           : launch(prefill_umma_kernel<__nv_bfloat16, 64>);
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

int pa_reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int64_t num_blocks, int32_t dtype,
                         void *stream) {
    int rc = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(key_cache, 16) ||
        !aligned(value_cache, 16) || !aligned(slot_mapping, 8))
        return PA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long num_slots = num_blocks * kBlock;
    const int vectors = num_kv_heads * (head_dim / 8);
    const dim3 grid(num_tokens, (vectors + kScatterThreads - 1) / kScatterThreads);
    if (grid.y > 65535) return PA_ERR_UNSUPPORTED;
    return launch_pdl(head_dim == 128 ? scatter_kernel<128> : scatter_kernel<64>, grid,
                      dim3(kScatterThreads), 0, st, static_cast<const uint4 *>(k),
                      static_cast<const uint4 *>(v), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), slot_mapping, num_kv_heads, num_slots);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_blocks_per_seq) {
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || block_size != kBlock ||
        max_blocks_per_seq <= 0)
        return 0;
    const int64_t parts = num_parts_for(max_blocks_per_seq);
    if (parts <= 1) return 0;
    return (size_t)workspace_layout(num_seqs, num_q_heads, head_dim, parts).total;
}

}  // extern "C"

namespace pa {
namespace {
// Host-side checks of a decode call's arguments, in the order pa_decode
// applies them (shared with pa_decode_static_workspace, so both return the
// same status for the same arguments).  PA_OK with *empty set means there is
// nothing to launch.
int check_decode_args(const void *out, const void *q, const void *key_cache,
                      const void *value_cache, const int32_t *block_tables,
                      const int32_t *context_lens, int32_t num_kv_heads, int32_t num_seqs,
                      int32_t num_q_heads, int32_t head_dim, int32_t block_size,
                      int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype, bool *empty) {
    *empty = false;
    int rc = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    if (group > 16) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) {
        *empty = true;
        return PA_OK;
    }
    if ((int64_t)num_seqs * num_q_heads >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned(key_cache, 16) || !aligned(value_cache, 16) || !aligned(q, 8) ||
        !aligned(out, 4) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PA_ERR_INVALID_ARG;
    if (num_parts_for(max_blocks_per_seq) > 8192) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// pa_decode, and pa_decode_append when k_new / v_new are given (arguments
// already checked, at least one sequence).
int decode_call(void *out, const void *q, const void *k_new, const void *v_new, void *key_cache,
                void *value_cache, const int32_t *block_tables, const int32_t *context_lens,
                int32_t num_kv_heads, float scale, int32_t num_seqs, int32_t num_q_heads,
                int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                int64_t num_blocks, int32_t dtype, void *workspace, size_t workspace_bytes,
                void *stream) {
    const int group = num_q_heads / num_kv_heads;
    const int64_t parts = num_parts_for(max_blocks_per_seq);

    DecodeArgs a;
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.ws_o = nullptr;
    a.ws_ml = nullptr;
    a.num_blocks = num_blocks;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_parts = (int)parts;
    a.part_blocks = part_blocks_for(max_blocks_per_seq);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.k_new = k_new;
    a.v_new = v_new;
    a.key_cache = key_cache;
    a.value_cache = value_cache;
    if (parts > 1) {
        const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                                     max_blocks_per_seq);
        if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
            return PA_ERR_WORKSPACE;
        const WorkspaceLayout l = workspace_layout(num_seqs, num_q_heads, head_dim, parts);
        char *base = static_cast<char *>(workspace);
        a.ws_o = reinterpret_cast<float *>(base + l.o_off);
        a.ws_ml = reinterpret_cast<float2 *>(base + l.ml_off);
    }
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, key_cache, num_blocks, num_kv_heads, head_dim, dtype) ||
        !encode_cache_map(&tmv, value_cache, num_blocks, num_kv_heads, head_dim, dtype))
        return PA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dtype == PA_F16 ? dispatch_decode<__half>(a, head_dim, group, tmk, tmv, st)
                           : dispatch_decode<__nv_bfloat16>(a, head_dim, group, tmk, tmv, st);
}
}  // namespace
}  // namespace pa

extern "C" {

int pa_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *context_lens, int32_t num_kv_heads,
              float scale, int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
              int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype,
              void *workspace, size_t workspace_bytes, void *stream) {
    bool empty = false;
    const int rc = check_decode_args(out, q, key_cache, value_cache, block_tables, context_lens,
                                     num_kv_heads, num_seqs, num_q_heads, head_dim, block_size,
                                     max_blocks_per_seq, num_blocks, dtype, &empty);
    if (rc != PA_OK || empty) return rc;
    return decode_call(out, q, nullptr, nullptr, const_cast<void *>(key_cache),
                       const_cast<void *>(value_cache), block_tables, context_lens, num_kv_heads,
                       scale, num_seqs, num_q_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, dtype, workspace, workspace_bytes, stream);
}

int pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                     void *key_cache, void *value_cache, const int32_t *block_tables,
                     const int32_t *context_lens, int32_t num_kv_heads, float scale,
                     int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t block_size,
                     int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype,
                     void *workspace, size_t workspace_bytes, void *stream) {
    bool empty = false;
    const int rc = check_decode_args(out, q, key_cache, value_cache, block_tables, context_lens,
                                     num_kv_heads, num_seqs, num_q_heads, head_dim, block_size,
                                     max_blocks_per_seq, num_blocks, dtype, &empty);
    if (rc != PA_OK || empty) return rc;
    if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return PA_ERR_INVALID_ARG;
    return decode_call(out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens,
                       num_kv_heads, scale, num_seqs, num_q_heads, head_dim, block_size,
                       max_blocks_per_seq, num_blocks, dtype, workspace, workspace_bytes, stream);
}

int pa_prefill_select(int32_t kernel) {
    if (kernel != PA_PREFILL_AUTO && kernel != PA_PREFILL_MMA_SYNC && kernel != PA_PREFILL_TCGEN05)
        return PA_ERR_INVALID_ARG;
    g_prefill_kernel.store(kernel);
    return PA_OK;
}

int pa_prefill(void *out, const void *q, const void *key_cache, const void *value_cache,
               const int32_t *block_tables, const int32_t *context_lens,
               const int32_t *query_start, int32_t max_query_len, int32_t num_kv_heads,
               float scale, int32_t num_seqs, int32_t num_q_heads, int32_t num_q_tokens,
               int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
               int64_t num_blocks, int32_t dtype, void *stream) {
    int rc = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_q_heads <= 0 || num_q_tokens < 0 || max_query_len < 0 ||
        max_blocks_per_seq <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    if (num_seqs == 0 || num_q_tokens == 0 || max_query_len == 0) return PA_OK;
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens ||
        !query_start)
        return PA_ERR_INVALID_ARG;
    if (!aligned(key_cache, 16) || !aligned(value_cache, 16) || !aligned(q, 4) ||
        !aligned(out, 4) || !aligned(block_tables, 4) || !aligned(context_lens, 4) ||
        !aligned(query_start, 4))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * num_kv_heads >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    const int which = g_prefill_kernel.load();
    const bool umma_ok = group <= kUmmaRows && aligned(q, 16) && aligned(out, 16) &&
                         scale > 0.f && scale < 3.0e38f;
    if (which == PA_PREFILL_TCGEN05 && !umma_ok) return PA_ERR_UNSUPPORTED;
    if (which != PA_PREFILL_MMA_SYNC && umma_ok) {
        const int urc = launch_prefill_umma(out, q, key_cache, value_cache, block_tables,
                                            context_lens, query_start, max_query_len, num_kv_heads,
                                            scale, num_seqs, num_q_heads, num_q_tokens, head_dim,
                                            max_blocks_per_seq, num_blocks, dtype,
                                            static_cast<cudaStream_t>(stream));
        if (urc != PA_ERR_UNSUPPORTED || which == PA_PREFILL_TCGEN05) return urc;
    }
    const int64_t tiles = ((int64_t)max_query_len * group + 63) / 64;
    if (tiles > 65535) return PA_ERR_UNSUPPORTED;
    constexpr int STAGES = 4;
    const size_t smem = (size_t)STAGES * 2 * kBlock * head_dim * 2 + 1024 +
                        (size_t)(head_dim == 128 ? prefill_q_bytes<128>() : prefill_q_bytes<64>()) +
                        (size_t)max_blocks_per_seq * 4;
    if (smem > 227 * 1024) return PA_ERR_UNSUPPORTED;
    PrefillArgs a;
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start = query_start;
    a.num_blocks = num_blocks;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_q_tokens = num_q_tokens;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.tiles_per_seq = 0;
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, key_cache, num_blocks, num_kv_heads, head_dim, dtype) ||
        !encode_cache_map(&tmv, value_cache, num_blocks, num_kv_heads, head_dim, dtype))
        return PA_ERR_CUDA;
    const dim3 grid(num_seqs * num_kv_heads, (unsigned)tiles);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto launch = [&](auto kernel) -> int {
        if (!set_smem(kernel, (int)smem)) return PA_ERR_CUDA;
        return launch_pdl(kernel, grid, dim3(128), smem, st, tmk, tmv, a);
    };
    if (dtype == PA_F16)
        return head_dim == 128 ? launch(prefill_mma_kernel<__half, 128, STAGES>)
                               : launch(prefill_mma_kernel<__half, 64, STAGES>);
    return head_dim == 128 ? launch(prefill_mma_kernel<__nv_bfloat16, 128, STAGES>)
                           : launch(prefill_mma_kernel<__nv_bfloat16, 64, STAGES>);
}

int pa_copy_blocks(void *key_cache, void *value_cache, const int32_t *src_dst_pairs,
                   int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   int64_t num_blocks, int32_t dtype, void *stream) {
    int rc = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !src_dst_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned(key_cache, 16) || !aligned(value_cache, 16) || !aligned(src_dst_pairs, 4))
        return PA_ERR_INVALID_ARG;
    const long long vec_per_block = (long long)num_kv_heads * kBlock * head_dim / 8;
    const int threads = 256;
    long long chunks = (vec_per_block + threads * 4 - 1) / (threads * 4);
    if (chunks > 65535) chunks = 65535;
    dim3 grid(num_pairs < 65535 ? num_pairs : 65535, (unsigned)chunks);
    return launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), src_dst_pairs, num_pairs, num_blocks,
                      vec_per_block);
}

int pa_swap_blocks(const void *src_key_cache, const void *src_value_cache, int64_t src_num_blocks,
                   void *dst_key_cache, void *dst_value_cache, int64_t dst_num_blocks,
                   const int32_t *src_dst_pairs, int32_t num_pairs, int32_t num_kv_heads,
                   int32_t head_dim, int32_t block_size, int32_t dtype, void *stream) {
    int rc = check_cache_shape(num_kv_heads, head_dim, block_size,
                               src_num_blocks > dst_num_blocks ? src_num_blocks : dst_num_blocks,
                               dtype);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!src_key_cache || !src_value_cache || !dst_key_cache || !dst_value_cache ||
        !src_dst_pairs)
        return PA_ERR_INVALID_ARG;
    for (int32_t p = 0; p < num_pairs; ++p) {
        const int64_t s = src_dst_pairs[2 * p], d = src_dst_pairs[2 * p + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) return PA_ERR_OUT_OF_RANGE;
    }
    const size_t block_bytes = (size_t)num_kv_heads * kBlock * head_dim * 2;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // One kernel over all pairs when every pool is device memory of this
    // device or mapped page-locked host memory (reached through its device
    // alias); otherwise one cudaMemcpyAsync per run of consecutive ids.
    const void *alias[4];
    const void *ptrs[4] = {src_key_cache, src_value_cache, dst_key_cache, dst_value_cache};
    bool kernel_path = true;
    for (int i = 0; i < 4 && kernel_path; ++i) kernel_path = device_alias(ptrs[i], &alias[i]);
    if (kernel_path) {
        const long long vec_per_block = (long long)block_bytes / 16;
        const int threads = 256;
        long long chunks = (vec_per_block + threads * 4 - 1) / (threads * 4);
        if (chunks > 65535) chunks = 65535;
        for (int32_t p0 = 0; p0 < num_pairs; p0 += kSwapChunk) {
            const int n = num_pairs - p0 < kSwapChunk ? num_pairs - p0 : kSwapChunk;
            SwapPairs pp;
            for (int i = 0; i < n; ++i)
                pp.p[i] = make_int2(src_dst_pairs[2 * (p0 + i)], src_dst_pairs[2 * (p0 + i) + 1]);
            const int rc2 = launch_pdl(
                swap_blocks_kernel, dim3(n, (unsigned)chunks), dim3(threads), 0, st,
                static_cast<const uint4 *>(alias[0]), static_cast<const uint4 *>(alias[1]),
                static_cast<uint4 *>(const_cast<void *>(alias[2])),
                static_cast<uint4 *>(const_cast<void *>(alias[3])), pp, n, vec_per_block);
            if (rc2 != PA_OK) return rc2;
        }
        return PA_OK;
    }
    const char *sk = static_cast<const char *>(src_key_cache);
    const char *sv = static_cast<const char *>(src_value_cache);
    char *dk = static_cast<char *>(dst_key_cache);
    char *dv = static_cast<char *>(dst_value_cache);
    for (int32_t p = 0; p < num_pairs;) {
        // extend a run while both ids advance by one
        int32_t q = p + 1;
        while (q < num_pairs && src_dst_pairs[2 * q] == src_dst_pairs[2 * (q - 1)] + 1 &&
               src_dst_pairs[2 * q + 1] == src_dst_pairs[2 * (q - 1) + 1] + 1)
            ++q;
        const size_t off_s = (size_t)src_dst_pairs[2 * p] * block_bytes;
        const size_t off_d = (size_t)src_dst_pairs[2 * p + 1] * block_bytes;
        const size_t n = (size_t)(q - p) * block_bytes;
        if (cudaMemcpyAsync(dk + off_d, sk + off_s, n, cudaMemcpyDefault, st) != cudaSuccess ||
            cudaMemcpyAsync(dv + off_d, sv + off_s, n, cudaMemcpyDefault, st) != cudaSuccess)
            return PA_ERR_CUDA;
        p = q;
    }
    return PA_OK;
}

int pa_get_error(void *stream, uint32_t *bits) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return PA_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
        return PA_ERR_CUDA;
    if (bits) *bits = word;
    if (!word) return PA_OK;
    return (word & PA_DEVERR_TIMEOUT) ? PA_ERR_TIMEOUT : PA_ERR_OUT_OF_RANGE;
}

int pa_selftest_wait_timeout(uint64_t timeout_ns, void *stream) {
    if (timeout_ns == 0 || timeout_ns > 1000000000ull) return PA_ERR_INVALID_ARG;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported shape or type";
        case PA_ERR_OUT_OF_RANGE: return "device saw an out-of-range index";
        case PA_ERR_NO_BLOCKS: return "no free blocks";
        case PA_ERR_CUDA: return "CUDA runtime error";
        case PA_ERR_WORKSPACE: return "workspace missing or too small";
        case PA_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

int pa_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------- no-allocation decode
// Scratch of pa_decode_static_workspace, for callers that cannot allocate
// device memory (see include/pa_api.h).  In host code `g_static_workspace`
// names a host-side stand-in, not a device address: its device address is
// looked up with cudaGetSymbolAddress, once per device and CUDA context, with
// that device current.
namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
struct StaticAddress {
    void *ptr;
    unsigned long long ctx_id;  // the context the address belongs to
};
StaticAddress g_static_address[kMaxDevices] = {};

// Device address of the array in the current device's current context.  A
// device reset (cudaDeviceReset) ends the context the cached address belongs
// to; the next call, in the new context, looks the address up again.
int static_workspace_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    StaticAddress &e = g_static_address[dev];
    const unsigned long long id = current_context_id();
    if (!e.ptr || id == 0 || id != e.ctx_id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return PA_ERR_CUDA;
        e.ptr = p;
        e.ctx_id = current_context_id();  // the lookup makes the primary context current
    }
    *out = e.ptr;
    return PA_OK;
}

}  // namespace

extern "C" int pa_decode_static_workspace(void *out, const void *q, const void *key_cache,
                                          const void *value_cache, const int32_t *block_tables,
                                          const int32_t *context_lens, int32_t num_kv_heads,
                                          float scale, int32_t num_seqs, int32_t num_q_heads,
                                          int32_t head_dim, int32_t block_size,
                                          int32_t max_blocks_per_seq, int64_t num_blocks,
                                          int32_t dtype, void *stream) {
    // the same argument checks as pa_decode, first, so both give the same
    // status for the same arguments; then the array's size
    bool empty = false;
    const int vrc = check_decode_args(out, q, key_cache, value_cache, block_tables, context_lens,
                                      num_kv_heads, num_seqs, num_q_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, dtype, &empty);
    if (vrc != PA_OK || empty) return vrc;
    const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                                 max_blocks_per_seq);
    if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0) {
        const int rc = static_workspace_address(&ws);
        if (rc != PA_OK) return rc;
    }
    return pa_decode(out, q, key_cache, value_cache, block_tables, context_lens, num_kv_heads,
                     scale, num_seqs, num_q_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, dtype, ws, need > 0 ? PA_STATIC_WORKSPACE_BYTES : 0, stream);
}
