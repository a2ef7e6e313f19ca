// 2^a on the FMA and integer pipes, for softmax weights.
//
// The special-function unit evaluates one ex2 per lane every few cycles; a
// softmax that needs an exponential per attention score can be bound by it.
// This evaluates 2^a with ordinary arithmetic instead (Cody-Waite style range
// reduction, then a polynomial), so part of the exponentials can run beside
// the ones on the special-function unit:
//   n = round(a)   (adding 1.5 * 2^23 leaves the rounded integer in the low
//                   mantissa bits), f = a - n in [-0.5, 0.5];
//   2^f ~ c0 + f (c1 + f (c2 + f c3)), the cubic fitted by least squares to
//         2^f on 2000 Chebyshev nodes of [-0.5, 0.5] with relative weights:
//         relative error below 8e-5 in float32 Horner evaluation, under the
//         rounding of the 16-bit P it feeds (2^-9 bf16, 2^-11 f16);
//   2^a = 2^f * 2^n, with 2^n built directly in the exponent field of 1.0;
//         the product is exact (2^f is in [0.7, 1.42] and n >= -125, so it
//         stays a normal number), and a NaN input stays NaN through it.
// Inputs are clamped at -125 so 2^n stays normal; 2^-125 (and anything
// below, masked scores included) then comes out as about 2^-125 rather than
// 0.  A softmax row's weight sum is at least 1 (its max scores 2^0), so such
// a weight is over 120 binary orders below it.  The clamp is a comparison
// that is false for NaN, so NaN is not clamped away.
#pragma once

#include <cstdint>
#include <cstring>

namespace pa {

constexpr float kExp2C0 = 0.999928951f;
constexpr float kExp2C1 = 0.693276227f;
constexpr float kExp2C2 = 0.242604047f;
constexpr float kExp2C3 = 0.055088684f;
constexpr float kExp2Round = 12582912.f;  // 1.5 * 2^23
constexpr float kExp2Min = -125.f;

#if defined(__CUDACC__)
#define PA_HD __host__ __device__
#else
#define PA_HD
#endif

PA_HD inline uint32_t f32_bits(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    return u;
}
PA_HD inline float f32_from(uint32_t u) {
    float x;
    memcpy(&x, &u, 4);
    return x;
}

// Scalar form: the same operations, in the same order, as exp2_fma_pair.
PA_HD inline float exp2_fma(float a) {
    a = a < kExp2Min ? kExp2Min : a;  // NaN passes (the comparison is false)
    const float nf = a + kExp2Round;
    const float n = nf - kExp2Round;
    const float f = fmaf(n, -1.f, a);
    const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
    // the low mantissa bits of nf hold n: shifted into the exponent field of
    // 1.0 they give 2^n
    return p * f32_from((f32_bits(nf) << 23) + 0x3f800000u);
}

#if defined(__CUDACC__)
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// exp2_fma on two values with paired (f32x2) arithmetic.
__device__ __forceinline__ void exp2_fma_pair(float a0, float a1, float &p0, float &p1) {
    const uint64_t a = f32x2_pack(a0 < kExp2Min ? kExp2Min : a0, a1 < kExp2Min ? kExp2Min : a1);
    const uint64_t nf = f32x2_add(a, f32x2_pack(kExp2Round, kExp2Round));
    const uint64_t n = f32x2_add(nf, f32x2_pack(-kExp2Round, -kExp2Round));
    const uint64_t f = f32x2_fma(n, f32x2_pack(-1.f, -1.f), a);
    uint64_t p = f32x2_fma(f32x2_pack(kExp2C3, kExp2C3), f, f32x2_pack(kExp2C2, kExp2C2));
    p = f32x2_fma(p, f, f32x2_pack(kExp2C1, kExp2C1));
    p = f32x2_fma(p, f, f32x2_pack(kExp2C0, kExp2C0));
    float m0, m1;
    f32x2_unpack(nf, m0, m1);
    const uint64_t two_n = f32x2_pack(__uint_as_float((__float_as_uint(m0) << 23) + 0x3f800000u),
                                      __uint_as_float((__float_as_uint(m1) << 23) + 0x3f800000u));
    f32x2_unpack(f32x2_mul(p, two_n), p0, p1);
}
#endif

}  // namespace pa
