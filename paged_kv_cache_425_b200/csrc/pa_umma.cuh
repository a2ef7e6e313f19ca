// Fifth-generation tensor-core (tcgen05) building blocks for sm_100a:
// tensor-memory (TMEM) allocation, the single-thread tcgen05.mma issue with
// shared-memory operand descriptors, completion through tcgen05.commit onto an
// mbarrier, and the warp-wide TMEM <-> register moves.
//
// Encodings follow the PTX ISA's tcgen05 chapter ("Shared memory descriptor",
// "Instruction descriptor" for .kind::f16).  The descriptor builders are
// constexpr host/device functions so host tests can check them.
#pragma once

#include <cstdint>

namespace pa {

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (64 bits):
//   [0,14)  matrix start address >> 4
//   [16,30) leading-dimension byte offset >> 4
//   [32,46) stride-dimension byte offset >> 4
//   [46,48) descriptor version, 1 on sm_100
//   [49,52) base offset (0: the swizzle atoms are 1024-byte aligned)
//   [52]    leading-dimension offset mode (0: byte offset)
//   [61,64) swizzle mode: 2 = 128-byte swizzle
// A 128-byte-swizzled operand is a stack of 8-row x 128-byte atoms, row r of
// an atom at r * 128 bytes with its 16-byte chunk c stored at chunk c ^ r.
//  * K-major (the reduction dimension contiguous): rows are M / N indices;
//    SBO = byte distance between 8-row groups; LBO is not used (set to 16).
//    Successive 16-element K steps inside the 128-byte row are addressed by
//    advancing the start address by 32 bytes.
//  * MN-major (M / N contiguous): each 128-byte row holds 64 M / N elements
//    of one K index; LBO = byte distance between 64-element M / N groups,
//    SBO = byte distance between groups of 8 K indices.
constexpr uint32_t kUmmaSwizzle128B = 2;

__host__ __device__ constexpr uint64_t umma_smem_desc(uint32_t smem_byte_addr, uint32_t lbo_bytes,
                                                      uint32_t sbo_bytes) {
    return (uint64_t)((smem_byte_addr >> 4) & 0x3FFFu) |
           ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) |
           ((uint64_t)kUmmaSwizzle128B << 61);
}

// Instruction descriptor of tcgen05.mma .kind::f16 (32 bits), dense, no
// negation, f32 accumulator:
//   [4,6)   D format: 1 = f32
//   [7,10)  A format, [10,13) B format: 0 = f16, 1 = bf16
//   [15]    A major (0 = K), [16] B major (0 = K, 1 = MN)
//   [17,23) N >> 3
//   [24,29) M >> 4
__host__ __device__ constexpr uint32_t umma_idesc_f16(uint32_t ab_format, uint32_t m, uint32_t n,
                                                      uint32_t b_mn_major) {
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_mn_major << 16) |
           ((n >> 3) << 17) | ((m >> 4) << 24);
}

#if defined(__CUDACC__)
// ---------------------------------------------------------------- TMEM
// Allocation and release are warp-wide and must be issued by the same warp.
// The allocated base address (lane 0, first column) is written to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Ordering of tcgen05 operations across a thread synchronisation (mbarrier
// or bar.sync): "before" on the signalling side, "after" on the waiting side.
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T per the descriptors; issued by one thread.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One arrival on `bar` once every tcgen05.mma this thread issued so far is
// complete (their shared-memory reads and TMEM writes included).
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
        : "memory");
}

// Warp-wide load of 32 lanes x N consecutive 32-bit columns starting at
// taddr (lane field = the warp's 32-lane quarter), completed before return.
#define PA_TMEM_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), \
                      "=r"(r[b + 4]), "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : PA_TMEM_R8(0), PA_TMEM_R8(8), PA_TMEM_R8(16), PA_TMEM_R8(24), PA_TMEM_R8(32),
          PA_TMEM_R8(40), PA_TMEM_R8(48), PA_TMEM_R8(56)
        : "r"(taddr)
        : "memory");
}

// The same for 128 columns.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
        "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
        "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
        "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
        "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : PA_TMEM_R8(0), PA_TMEM_R8(8), PA_TMEM_R8(16), PA_TMEM_R8(24), PA_TMEM_R8(32),
          PA_TMEM_R8(40), PA_TMEM_R8(48), PA_TMEM_R8(56), PA_TMEM_R8(64), PA_TMEM_R8(72),
          PA_TMEM_R8(80), PA_TMEM_R8(88), PA_TMEM_R8(96), PA_TMEM_R8(104), PA_TMEM_R8(112),
          PA_TMEM_R8(120)
        : "r"(taddr)
        : "memory");
}

// The same for 32 columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : PA_TMEM_R8(0), PA_TMEM_R8(8), PA_TMEM_R8(16), PA_TMEM_R8(24)
        : "r"(taddr)
        : "memory");
}
#undef PA_TMEM_R8

// Warp-wide stores of 32 lanes x N columns; the caller waits with
// tmem_wait_st() before signalling the stored values to another thread.
#define PA_TMEM_W8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), \
                      "r"(r[b + 4]), "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])
// 32 columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        PA_TMEM_W8(0), PA_TMEM_W8(8), PA_TMEM_W8(16), PA_TMEM_W8(24)
        : "memory");
}

// The same for 16 columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        PA_TMEM_W8(0), PA_TMEM_W8(8)
        : "memory");
}
#undef PA_TMEM_W8

// D[tmem] (+)= A[tmem] * B[smem]^T: A is read from tensor memory (M lanes,
// K 16-bit elements packed two per 32-bit column, the lower index in the low
// half), B through its shared-memory descriptor; issued by one thread.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
#endif  // __CUDACC__

}  // namespace pa
