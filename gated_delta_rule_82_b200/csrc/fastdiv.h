// fastdiv.h -- division by a divisor fixed for a whole launch, as one multiply-high, one add and
// one shift (the round-up method of T. Granlund and P. Montgomery, "Division by Invariant
// Integers using Multiplication", PLDI 1994, section 4).  For a divisor d >= 1 take
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1 (which fits in 32 bits); then every
// 32-bit n has  n / d = (mulhi(m, n) + n) >> l, with the sum formed in 64 bits.
//
// Plain C++ (no CUDA types), so that host code and a host-side test can use the same
// definitions as the kernels.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define CKDA_HD __host__ __device__ __forceinline__
#else
#define CKDA_HD inline
#endif

namespace ckda {

struct FastDiv {
    uint32_t d;   // the divisor
    uint32_t m;   // multiplier
    uint32_t l;   // shift
};

// Parameters for divisor d (d >= 1; d = 0 gives the divisor 1).
inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d ? d : 1u;
    f.l = 0;
    while ((1ull << f.l) < f.d) ++f.l;
    f.m = (uint32_t)((((1ull << 32) * ((1ull << f.l) - f.d)) / f.d) + 1ull);
    return f;
}

CKDA_HD uint32_t fastdiv(const FastDiv& f, uint32_t n) {
#ifdef __CUDA_ARCH__
    const uint64_t hi = __umulhi(f.m, n);
#else
    const uint64_t hi = ((uint64_t)f.m * n) >> 32;
#endif
    return (uint32_t)((hi + n) >> f.l);
}

}  // namespace ckda
