// Philox4x32-10 counter-based random numbers (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011): a 128-bit counter and
// a 64-bit key through 10 rounds of two 32x32 -> 64-bit multiplies and xors, the
// key bumped by two Weyl constants between rounds. Used for the Gumbel noise of
// the sampled drafter, where the uniforms cannot be passed in (one per vocabulary
// entry and block position).
#pragma once

#include <stdint.h>

namespace dfl {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;   // round multipliers
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;   // key increments
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint32_t hi0 = __umulhi(kM0, c.x), lo0 = kM0 * c.x;
    const uint32_t hi1 = __umulhi(kM1, c.z), lo1 = kM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// A 32-bit word to a uniform strictly inside (0, 1): ((w >> 9) + 1/2) / 2^23,
// exact in fp32.
__device__ __forceinline__ float philox_uniform(uint32_t w) {
  return ((float)(w >> 9) + 0.5f) * (1.0f / 8388608.0f);
}

}  // namespace dfl
