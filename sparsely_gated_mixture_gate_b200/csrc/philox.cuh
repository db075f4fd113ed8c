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
// in [0,1).  r = sqrt(-2 ln u1); z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).
// Both transcendentals use that their arguments are 24-bit integers:
//  * ln u1 = (e - 24) ln 2 + ln g, with the integer 2^(e) g (g in
//    [sqrt(1/2), sqrt 2)) read off its exact float, and ln g = 2 atanh(s),
//    s = (g - 1) / (g + 1), |s| < 0.1716, by the series 2 (s + s^3/3 + ... +
//    s^9/9) (truncation below 4e-10 relative).  Relative error of ln u1 at
//    most 2.1e-7 over all 2^24 inputs with a correctly rounded quotient s (the
//    approximate quotient used adds at most 2 ulp of s, 2.4e-7 relative);
//    u1 = 1 gives ln = 0 exactly.
//  * the quarter turn nearest to u2 comes from its top two bits and the
//    remainder f in [-1/2, 1/2) of a quarter turn is exact; sin(pi f / 2) and
//    cos(pi f / 2) by their Taylor series to degree 9 and 8 (truncation below
//    3e-8), then turned by the quarter turns.  Absolute error at most 8.9e-8
//    over all 2^24 inputs.
__device__ __forceinline__ void box_muller2(uint32_t w0, uint32_t w1, float &z0, float &z1) {
  // ---- r = sqrt(-2 ln u1)
  const uint32_t b = __float_as_uint((float)((w0 >> 8) + 1u));  // exact: at most 2^24
  const uint32_t mant = b & 0x7fffffu;
  const bool big = mant >= 0x3504f3u;  // mantissa >= sqrt 2: halve g, raise the exponent
  const int e = (int)(b >> 23) - 127 - 24 + (big ? 1 : 0);
  const float g = __uint_as_float(mant | (big ? 0x3f000000u : 0x3f800000u));
  const float s = __fdividef(g - 1.0f, g + 1.0f);
  const float s2 = s * s;
  float p = 2.0f / 9.0f;
  p = fmaf(p, s2, 2.0f / 7.0f);
  p = fmaf(p, s2, 2.0f / 5.0f);
  p = fmaf(p, s2, 2.0f / 3.0f);
  p = fmaf(p, s2, 2.0f);
  const float lnu = fmaf((float)e, 0.6931471805599453f, p * s);
  const float r = sqrtf(-2.0f * lnu);
  // ---- cos and sin of 2 pi u2
  const uint32_t jr = (w1 >> 8) + (1u << 21);  // rounded to the nearest quarter turn
  const uint32_t quad = (jr >> 22) & 3u;
  const float f = (float)((int)(jr & 0x3fffffu) - (1 << 21)) * 2.384185791015625e-7f;  // 2^-22
  const float f2 = f * f;
  float sn = 0.00016044118478735975f;  // (pi/2)^9 / 9!
  sn = fmaf(sn, f2, -0.004681754135318687f);
  sn = fmaf(sn, f2, 0.07969262624616703f);
  sn = fmaf(sn, f2, -0.6459640975062462f);
  sn = fmaf(sn, f2, 1.5707963267948966f);
  sn *= f;
  float cs = 0.0009192602748394263f;  // (pi/2)^8 / 8!
  cs = fmaf(cs, f2, -0.020863480763352957f);
  cs = fmaf(cs, f2, 0.253669507901048f);
  cs = fmaf(cs, f2, -1.2337005501361697f);
  cs = fmaf(cs, f2, 1.0f);
  const bool odd = (quad & 1u) != 0u;
  const float c0 = odd ? sn : cs, s0 = odd ? cs : sn;
  z0 = r * (((quad + 1u) & 2u) ? -c0 : c0);
  z1 = r * ((quad & 2u) ? -s0 : s0);
}

}  // namespace moe
