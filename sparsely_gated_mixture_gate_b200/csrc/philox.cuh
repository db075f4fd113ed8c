// philox.cuh -- the gate's StandardNormal() source on the device.
//
// Philox4x32-10 as defined by Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3" (SC'11): ten rounds, each multiplying words 0
// and 2 by the two round multipliers, exchanging the product halves across the
// words and folding in the key, which is bumped by the two Weyl constants
// between rounds.  Box-Muller (Box & Muller 1958) turns two words into two
// independent standard normal deviates (its cosine and sine branches).
//
// Stream convention (the pages only say "StandardNormal()", [SGMoE-xyz]
// "Noisy Top-K 門控"): key (seed lo, seed hi), counter (token, expert/4,
// gate id, 0); words (0,1) give the cosine and sine branches of one
// Box-Muller transform for experts 4m and 4m+1, words (2,3) those of a second
// transform for experts 4m+2 and 4m+3.
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
// in [0,1); both exact in fp32.  r = sqrt(-2 ln u1); z0 = r cos(2 pi u2),
// z1 = r sin(2 pi u2).
__device__ __forceinline__ void box_muller2(uint32_t w0, uint32_t w1, float &z0, float &z1) {
  const float u1 = (float)((w0 >> 8) + 1u) * 5.9604644775390625e-8f;  // 2^-24
  const float u2 = (float)(w1 >> 8) * 5.9604644775390625e-8f;
  const float r = sqrtf(-2.0f * logf(u1));
  float sn, cs;
  sincospif(2.0f * u2, &sn, &cs);
  z0 = r * cs;
  z1 = r * sn;
}

}  // namespace moe
