// Host-side check of the kernels' division by a launch-invariant divisor (csrc/fastdiv.h)
// against the machine's own integer division: every n < 4096 for every divisor below 4096, the
// 32-bit edges, powers of two and their neighbours, and random pairs.  Prints the number of
// mismatches; exits nonzero if there is any.
#include <cstdio>
#include <random>

#include "fastdiv.h"

int main() {
    std::mt19937_64 rng(20241202);
    long bad = 0, checked = 0;
    auto check = [&](uint32_t d, uint32_t n) {
        const ckda::FastDiv f = ckda::make_fastdiv(d);
        if (ckda::fastdiv(f, n) != n / d) {
            if (bad < 5) std::printf("mismatch d=%u n=%u\n", d, n);
            ++bad;
        }
        ++checked;
    };
    for (uint32_t d = 1; d < 4096; ++d) {
        for (uint32_t n = 0; n < 4096; ++n) check(d, n);
        for (uint32_t n : {0x7fffffffu, 0x80000000u, 0xfffffffeu, 0xffffffffu}) check(d, n);
    }
    for (int s = 0; s < 32; ++s)
        for (int k = -2; k <= 2; ++k) {
            const uint32_t d = (1u << s) + (uint32_t)k;
            if (d == 0 || (s == 31 && k > 0 && d < (1u << 31))) continue;
            for (uint32_t n : {0u, 1u, d - 1, d, d + 1, 2 * d - 1, 2 * d, 0xfffffffeu, 0xffffffffu})
                check(d, n);
        }
    for (int k = 0; k < 4000000; ++k) {
        uint32_t d = (uint32_t)(rng() >> (32 + rng() % 32));
        if (d == 0) d = 1;
        check(d, (uint32_t)rng());
    }
    std::printf("checked %ld mismatches %ld\n", checked, bad);
    return bad != 0;
}
