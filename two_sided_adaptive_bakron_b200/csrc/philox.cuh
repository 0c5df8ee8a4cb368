// philox.cuh -- Philox4x64-10, the counter-based generator of the stochastic-rounding variates
// (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011,
// section 4: Philox with N = 4 words of 64 bits and R = 10 rounds).
//
// Each round multiplies words 0 and 2 by the round multipliers (full 128-bit products), xors
// the high halves with words 1 and 3 and with the round key, and permutes: the new words are
// (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0)). The key advances by the
// Weyl increments (golden ratio and sqrt(3) - 1 in 64-bit fixed point) between rounds.
#pragma once

#include <cstdint>

namespace bakron {

__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                              uint64_t k0, uint64_t k1, uint64_t (&out)[4]) {
    constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;
    constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull, kW1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t hi0 = __umul64hi(kM0, c0), lo0 = kM0 * c0;
        const uint64_t hi1 = __umul64hi(kM1, c2), lo1 = kM1 * c2;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += kW0;
        k1 += kW1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

}  // namespace bakron
