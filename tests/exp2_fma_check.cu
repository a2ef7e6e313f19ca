// Host check of the FMA-pipe 2^a used by the tcgen05 prefill softmax
// (pa_exp2.cuh, scalar form; the paired device form runs the same operations
// in the same order).  Prints "ok" when, over a dense grid of a in [-125, 8],
// the relative error against the double-precision 2^a stays below 1e-4,
// every a below -125 gives a value in (0, 2^-124], and NaN gives NaN.
#include <cmath>
#include <cstdio>

#include "pa_exp2.cuh"

int main() {
    double worst = 0.0, at = 0.0;
    for (long i = 0; i <= 1330000; ++i) {
        const float a = -125.f + (float)i * 1e-4f;
        if (a > 8.f) break;
        const double rel = std::fabs((double)pa::exp2_fma(a) / std::exp2((double)a) - 1.0);
        if (rel > worst) {
            worst = rel;
            at = a;
        }
    }
    bool ok = worst < 1e-4;
    const float low[] = {-125.5f, -200.f, -1e29f, -3.0e38f};
    for (float a : low) {
        const float p = pa::exp2_fma(a);
        ok = ok && p > 0.f && p <= std::ldexp(1.f, -124);
    }
    // NaN stays NaN: the clamp must not turn it into a tiny weight
    ok = ok && std::isnan(pa::exp2_fma(std::nanf(""))) && std::isnan(pa::exp2_fma(-std::nanf("")));
    // exact powers of two come out within the polynomial's error of 2^n
    for (int n = -120; n <= 8; ++n) {
        const double rel = std::fabs((double)pa::exp2_fma((float)n) / std::ldexp(1.0, n) - 1.0);
        ok = ok && rel < 1e-4;
    }
    std::printf("%s worst %.3g at %.4f\n", ok ? "ok" : "FAIL", worst, at);
    return ok ? 0 : 1;
}
