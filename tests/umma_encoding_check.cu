// Host-only cross-check of the tcgen05 descriptor encodings in pa_umma.cuh
// against CUTLASS's definitions of the same fields (cute/arch/mma_sm100_desc.hpp):
// the instruction descriptor from cute::UMMA::make_instr_desc, and the
// shared-memory descriptor assembled from cute::UMMA::SmemDescriptor's
// bitfields.  Prints "ok" and exits 0 when every case agrees.
#include <cstdint>
#include <cstdio>

#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>

#include "pa_umma.cuh"

namespace U = cute::UMMA;

template <class T, int M, int N, U::Major BM>
static uint32_t theirs_idesc() {
    return static_cast<uint32_t>(U::make_instr_desc<T, T, float, M, N, U::Major::K, BM>());
}

int main() {
    int bad = 0;
    auto chk = [&](uint64_t mine, uint64_t ref, const char *what) {
        if (mine != ref) {
            std::printf("mismatch %s: %llx vs %llx\n", what, (unsigned long long)mine,
                        (unsigned long long)ref);
            ++bad;
        }
    };
    // Q K^T (both K-major) and P V (V MN-major), N = 128 / 64, f16 and bf16
    chk(pa::umma_idesc_f16(1, 128, 128, 0), theirs_idesc<cute::bfloat16_t, 128, 128, U::Major::K>(), "bf16 M128 N128 K/K");
    chk(pa::umma_idesc_f16(1, 128, 128, 1), theirs_idesc<cute::bfloat16_t, 128, 128, U::Major::MN>(), "bf16 M128 N128 K/MN");
    chk(pa::umma_idesc_f16(1, 128, 64, 1), theirs_idesc<cute::bfloat16_t, 128, 64, U::Major::MN>(), "bf16 M128 N64 K/MN");
    chk(pa::umma_idesc_f16(0, 128, 128, 0), theirs_idesc<cute::half_t, 128, 128, U::Major::K>(), "f16 M128 N128 K/K");
    chk(pa::umma_idesc_f16(0, 128, 128, 1), theirs_idesc<cute::half_t, 128, 128, U::Major::MN>(), "f16 M128 N128 K/MN");
    chk(pa::umma_idesc_f16(0, 128, 64, 1), theirs_idesc<cute::half_t, 128, 64, U::Major::MN>(), "f16 M128 N64 K/MN");

    const uint32_t addrs[] = {0x400, 0x8420, 0x12360, 0x37ff0};
    const uint32_t lbos[] = {16, 2048, 16384};
    const uint32_t sbos[] = {1024, 8192};
    for (uint32_t a : addrs)
        for (uint32_t l : lbos)
            for (uint32_t s : sbos) {
                U::SmemDescriptor d;
                d.desc_ = 0;
                d.start_address_ = static_cast<uint16_t>(a >> 4);
                d.leading_byte_offset_ = static_cast<uint16_t>(l >> 4);
                d.stride_byte_offset_ = static_cast<uint16_t>(s >> 4);
                d.version_ = 1;
                d.base_offset_ = 0;
                d.lbo_mode_ = 0;
                d.layout_type_ = static_cast<uint8_t>(U::LayoutType::SWIZZLE_128B);
                chk(pa::umma_smem_desc(a, l, s), d.desc_, "smem descriptor");
            }
    std::printf(bad ? "FAIL\n" : "ok\n");
    return bad != 0;
}
