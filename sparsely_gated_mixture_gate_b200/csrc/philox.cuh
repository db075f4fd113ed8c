// philox.cuh -- the gate's StandardNormal() source on the device.
//
// Philox4x32-10 as defined by Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3" (SC'11): ten rounds, each multiplying words 0
// and 2 by the two round multipliers, exchanging the product halves across the
// words and folding in the key, which is bumped by the two Weyl constants
// between rounds.  Box-Muller (Box & Muller 1958), cosine branch, turns two
// words into one standard normal deviate.
//
// Stream convention (the pages only say "StandardNormal()", [SGMoE-xyz]
// "Noisy Top-K 門控"): key (seed lo, seed hi), counter (token, expert/2,
// gate id, 0); words (0,1) feed the even expert of the pair, (2,3) the odd one.
#pragma once
#include <stdint.h>

namespace moe {

__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, ctr.x), lo0 = 0xD2511F53u * ctr.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, ctr.z), lo1 = 0xCD9E8D57u * ctr.z;
    ctr = make_uint4(hi1 ^ ctr.y ^ k0, lo1, hi0 ^ ctr.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return ctr;
}

// u1 = (top 24 bits of w0 + 1) / 2^24 in (0,1], u2 = (top 24 bits of w1) / 2^24
// in [0,1); both exact in fp32.  eps = sqrt(-2 ln u1) cos(2 pi u2).
__device__ __forceinline__ float box_muller(uint32_t w0, uint32_t w1) {
  const float u1 = (float)((w0 >> 8) + 1u) * 5.9604644775390625e-8f;  // 2^-24
  const float u2 = (float)(w1 >> 8) * 5.9604644775390625e-8f;
  return sqrtf(-2.0f * logf(u1)) * cospif(2.0f * u2);
}

}  // namespace moe
