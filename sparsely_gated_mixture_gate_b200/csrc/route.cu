// route.cu -- per-token routing decisions and the smoothed load.
//
// For every row (one token under one gate):
//   H_i = c_i + eps_i * s_i            ([SGMoE-xyz] "Noisy Top-K 門控")
//   top-(k+1) of H, larger first, ties to the lower index
//   G = Softmax(KeepTopK(H, k))        (softmax over the kept k)
//   P(x,i) = Phi((c_i - kth_excluding(H,k,i)) / s_i)   ([SGMoE-xyz] "負載平衡損失")
//     kth_excluding is the (k+1)-th largest H when i is kept, the k-th otherwise
//   Switch router ([MoE-deep] §3.1): p = softmax(c) over all experts, the row
//   goes to argmax p with gate p_argmax; sum_t p_i is accumulated too.
// One warp per row; each lane scans column pairs (2m, 2m+1), which share one
// Philox call.  Each lane keeps a sorted top-(k+1) list in registers and the
// warp merges the 32 lists with shuffles.  Column sums of P (and of p) are
// accumulated per warp in shared memory, summed over the 4 warps in fixed
// order, and written per tile; route_reduce sums the tiles in fixed order,
// so the load is bitwise reproducible.
#include <float.h>
#include <limits.h>

#include "internal.h"
#include "philox.cuh"

namespace moe {
namespace {

constexpr int NW = 4;  // warps per routing block

struct Cand {
  float v;
  int i;
};

// a ranks before b: larger value first, equal values -> lower index first.
// NaN never ranks before anything.
__device__ __forceinline__ bool before(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

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

template <int K1>
__global__ void __launch_bounds__(NW * 32) route_kernel(RouteArgs a) {
  extern __shared__ float smem[];
  const int nb = a.nb;
  float *part = smem;                                   // [NW][nb]
  float *psum = a.psum_part ? smem + NW * nb : nullptr; // [NW][nb]

  // ---- which group, which rows
  const int tile = blockIdx.x;
  int g = 0, row0, row_end;
  if (a.seg_tiles) {
    if (tile >= a.seg_tiles[a.G]) return;
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.seg_tiles[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    row0 = a.seg_off[g] + (tile - a.seg_tiles[g]) * a.RT;
    row_end = min(row0 + a.RT, a.seg_off[g + 1]);
  } else {
    row0 = tile * a.RT;
    row_end = min(row0 + a.RT, a.R);
  }

  for (int i = threadIdx.x; i < NW * nb * (psum ? 2 : 1); i += NW * 32) smem[i] = 0.f;
  __syncthreads();

  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = a.k;
  const uint32_t key0 = (uint32_t)(a.seed & 0xffffffffu), key1 = (uint32_t)(a.seed >> 32);
  const uint32_t gate_id = a.secondary ? (uint32_t)(1 + g) : 0u;
  float *mypart = part + w * nb;
  float *mypsum = psum ? psum + w * nb : nullptr;
  bool bad = false;

  for (int row = row0 + w; row < row_end; row += NW) {
    const int t = a.row_token ? a.row_token[row] : row;
    const float *crow = a.c + (size_t)row * nb;
    const float *srow = a.s + (size_t)row * nb;

    Cand L[K1];
#pragma unroll
    for (int j = 0; j < K1; ++j) { L[j].v = -INFINITY; L[j].i = INT_MAX; }
    float mx = -INFINITY, se = 0.f;  // online softmax of c (Switch)

    // ---- pass 1: noisy logits, per-lane top-(k+1)
    for (int m = lane; 2 * m < nb; m += 32) {
      const int i0 = 2 * m, i1 = 2 * m + 1;
      const bool has1 = i1 < nb;
      const float c0 = crow[i0], c1 = has1 ? crow[i1] : 0.f;
      float h0 = c0, h1 = c1;
      if (a.noise) {
        const uint4 wd = philox4x32_10(make_uint4((uint32_t)t, (uint32_t)m, gate_id, 0u), key0, key1);
        const float s0 = srow[i0], s1 = has1 ? srow[i1] : 0.f;
        h0 = fmaf(box_muller(wd.x, wd.y), s0, c0);
        h1 = fmaf(box_muller(wd.z, wd.w), s1, c1);
      }
      bad |= !isfinite(h0) || (has1 && !isfinite(h1));
      insert<K1>(L, h0, i0);
      if (has1) insert<K1>(L, h1, i1);
      if (a.router == MOE_ROUTER_SWITCH) {
        const float m2 = fmaxf(mx, has1 ? fmaxf(c0, c1) : c0);
        se = se * expf(mx - m2) + expf(c0 - m2) + (has1 ? expf(c1 - m2) : 0.f);
        mx = m2;
      }
    }

    // ---- warp merge: K1 rounds of a warp-wide arg-max with the same order
    Cand S[K1];
#pragma unroll
    for (int r = 0; r < K1; ++r) {
      float bv = L[0].v;
      int bi = L[0].i;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (before(ov, oi, bv, bi)) { bv = ov; bi = oi; }
      }
      S[r].v = bv;
      S[r].i = bi;
      if (L[0].i == bi && bi != INT_MAX) {  // the owner pops its head
#pragma unroll
        for (int j = 0; j < K1 - 1; ++j) L[j] = L[j + 1];
        L[K1 - 1].v = -INFINITY;
        L[K1 - 1].i = INT_MAX;
      }
    }

    // ---- gates
    float M = 0.f, SE = 1.f;
    if (a.router == MOE_ROUTER_SWITCH) {
      M = mx; SE = se;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, M, off);
        const float os = __shfl_xor_sync(0xffffffffu, SE, off);
        const float m2 = fmaxf(M, om);
        const float a1 = (M == -INFINITY) ? 0.f : SE * expf(M - m2);
        const float a2 = (om == -INFINITY) ? 0.f : os * expf(om - m2);
        M = m2;
        SE = a1 + a2;
      }
    }
    float gate_j = 0.f;
    int idx_j = 0;
    {
      float den = 0.f;
#pragma unroll
      for (int j = 0; j < K1 - 1; ++j)
        if (j < k) den += expf(S[j].v - S[0].v);
#pragma unroll
      for (int j = 0; j < K1 - 1; ++j)
        if (j == lane) {
          idx_j = S[j].i;
          gate_j = (a.router == MOE_ROUTER_SWITCH) ? expf(crow[S[0].i] - M) / SE
                                                   : expf(S[j].v - S[0].v) / den;
        }
    }
    if (lane < k) {
      int slot = lane, outrow = t;
      float gmul = 1.f;
      int ebase = 0;
      if (a.secondary) {
        const int ps = a.row_slot[row];
        slot = ps * k + lane;
        gmul = a.gate_mult[(size_t)t * a.k1 + ps];
        ebase = g * a.expert_stride;
      }
      a.out_idx[(size_t)outrow * a.K + slot] = ebase + idx_j;
      a.out_gate[(size_t)outrow * a.K + slot] = gmul * gate_j;
    }

    // ---- pass 2: smoothed load (and Switch probabilities)
    const float thr_kept = S[K1 - 1].v;  // (k+1)-th largest, -inf if it does not exist
    const float thr_out = S[K1 - 2].v;   // k-th largest
    for (int i = lane; i < nb; i += 32) {
      bool kept = false;
#pragma unroll
      for (int j = 0; j < K1 - 1; ++j) kept |= (S[j].i == i) && (j < k);
      float P;
      if (!a.noise) {
        P = kept ? 1.f : 0.f;
      } else {
        const float thr = kept ? thr_kept : thr_out;
        const float ci = crow[i], si = srow[i];
        if (thr == -INFINITY) P = 1.f;
        else if (si == 0.f) P = ci > thr ? 1.f : (ci < thr ? 0.f : 0.5f);
        else P = normcdff((ci - thr) / si);
      }
      mypart[i] += P;
      if (mypsum) mypsum[i] += expf(crow[i] - M) / SE;
    }
  }
  if (bad && a.status) atomicOr(a.status, MOE_STATUS_NONFINITE);

  __syncthreads();
  float *outp = a.load_part + (size_t)tile * nb;
  for (int i = threadIdx.x; i < nb; i += NW * 32) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) sum += part[q * nb + i];
    outp[i] = sum;
  }
  if (psum) {
    float *outq = a.psum_part + (size_t)tile * nb;
    for (int i = threadIdx.x; i < nb; i += NW * 32) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < NW; ++q) sum += psum[q * nb + i];
      outq[i] = sum;
    }
  }
}

__global__ void route_reduce_kernel(const float *part, const int *seg_tiles, int ntiles_flat,
                                    int nb, float *out) {
  const int g = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= nb) return;
  const int t0 = seg_tiles ? seg_tiles[g] : 0;
  const int t1 = seg_tiles ? seg_tiles[g + 1] : ntiles_flat;
  float sum = 0.f;
  for (int t = t0; t < t1; ++t) sum += part[(size_t)t * nb + j];
  out[(size_t)g * nb + j] = sum;
}

__global__ void hier_load_kernel(const float *load_p, const float *load2, const int *cnt, int a,
                                 int b, float *load) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a * b) return;
  const int g = e / b;
  const int c = cnt[g];
  load[e] = c > 0 ? load_p[g] * load2[e] / (float)c : 0.f;
}

}  // namespace

int launch_route(const RouteArgs &a, int tiles_upper, cudaStream_t st) {
  const size_t smem = sizeof(float) * NW * a.nb * (a.psum_part ? 2 : 1);
  static bool attr_done[kMaxK + 2] = {};
  auto go = [&](auto kern, int K1) -> int {
    if (!attr_done[K1]) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      attr_done[K1] = true;
    }
    return launch("route_topk", kern, dim3(tiles_upper), dim3(NW * 32), smem, st, a);
  };
  switch (a.k + 1) {
    case 2: return go(route_kernel<2>, 2);
    case 3: return go(route_kernel<3>, 3);
    case 4: return go(route_kernel<4>, 4);
    case 5: return go(route_kernel<5>, 5);
    case 6: return go(route_kernel<6>, 6);
    case 7: return go(route_kernel<7>, 7);
    case 8: return go(route_kernel<8>, 8);
    case 9: return go(route_kernel<9>, 9);
    default: return MOE_EINVAL;
  }
}

int launch_route_reduce(const float *part, const int *seg_tiles, int G, int ntiles_flat, int nb,
                        float *out, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(nb, 256), G);
  return launch("route_reduce", route_reduce_kernel, grid, dim3(256), 0, st, part, seg_tiles,
                ntiles_flat, nb, out);
}

int launch_hier_load(const float *load_p, const float *load2, const int *cnt, int a, int b,
                     float *load, cudaStream_t st) {
  return launch("hier_load", hier_load_kernel, dim3((unsigned)ceil_div((int64_t)a * b, 256)),
                dim3(256), 0, st, load_p, load2, cnt, a, b, load);
}

}  // namespace moe
