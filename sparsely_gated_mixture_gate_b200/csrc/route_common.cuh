// route_common.cuh -- the routing kernels' ranking order and candidate lists.
//
// KeepTopK ([SGMoE-xyz] "Noisy Top-K 門控") keeps the k largest H of a row;
// equal values rank by the lower expert index, and NaN ranks before nothing.
#pragma once
#include <limits.h>
#include <stdint.h>

namespace moe {

struct Cand {
  float v;
  int i;
};

// a ranks before b: larger value first, equal values -> lower index first.
// NaN never ranks before anything.
__device__ __forceinline__ bool before(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

// insert (v, i) into a list sorted by before(), dropping the last entry
template <int K1>
__device__ __forceinline__ void insert(Cand (&L)[K1], float v, int i) {
  if (!before(v, i, L[K1 - 1].v, L[K1 - 1].i)) return;
#pragma unroll
  for (int j = K1 - 1; j >= 0; --j) {
    const bool gt = before(v, i, L[j].v, L[j].i);
    const bool gt_prev = (j > 0) ? before(v, i, L[j - 1].v, L[j - 1].i) : false;
    if (gt) {
      if (gt_prev) L[j] = L[j - 1];
      else { L[j].v = v; L[j].i = i; }
    }
  }
}

}  // namespace moe
