// philox.cuh -- Philox4x32-10 counter-based generator, written from its
// published definition (Salmon, Moraes, Dror & Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11, Sec. 4): each of the 10 rounds takes
// two 32x32->64-bit products of counter words with fixed multipliers, swaps
// and xors the halves with the round key, and the 2-word key advances by a
// Weyl sequence between rounds.
#pragma once

#include <stdint.h>

namespace wildcat {

struct Philox4x32 {
    static constexpr uint32_t kMul0 = 0xD2511F53u;
    static constexpr uint32_t kMul1 = 0xCD9E8D57u;
    static constexpr uint32_t kWeyl0 = 0x9E3779B9u;  // golden ratio
    static constexpr uint32_t kWeyl1 = 0xBB67AE85u;  // sqrt(3) - 1

    __device__ __forceinline__ static uint4 block(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
        for (int round = 0; round < 10; ++round) {
            const uint32_t hi0 = __umulhi(kMul0, c.x), lo0 = kMul0 * c.x;
            const uint32_t hi1 = __umulhi(kMul1, c.z), lo1 = kMul1 * c.z;
            c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
            k0 += kWeyl0;
            k1 += kWeyl1;
        }
        return c;
    }
};

// Uniform in (0, 1] that draws pivot `step` of instance `inst`:
// counter (step, inst, 0, 0), key (seed_lo, seed_hi), top 53 bits of (x1:x0).
__device__ __forceinline__ double pivot_uniform(uint64_t seed, uint32_t step, uint32_t inst) {
    const uint4 x = Philox4x32::block(make_uint4(step, inst, 0u, 0u), (uint32_t)seed,
                                      (uint32_t)(seed >> 32));
    const uint64_t bits = ((((uint64_t)x.y) << 32) | (uint64_t)x.x) >> 11;
    return ((double)bits + 1.0) * 0x1.0p-53;
}

}  // namespace wildcat
