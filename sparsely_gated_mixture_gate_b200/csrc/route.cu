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
//   Sigmoid router ([MoE-deep] §6.2, §6.3): H_i = c_i + b_i with the selection
//   bias b, top-k of H, gates Sigmoid(c_i) / sum of Sigmoid(c_j) over the kept.
//   Router statistics ([MoE-intro] 第三部分, optional): per row |c|^2 and the
//   entropy of softmax(c), summed over the tile's rows in a fixed order.
// Pass 1, one warp per row (rows of at most 128 columns: four rows per warp, 8
// lanes each; against two rows of 16 lanes, the rounds and their barriers
// halve: 8-26% faster, most where the tiles are short): each lane scans
// column quads 4m .. 4m+3 (16-byte
// loads, one Philox call per quad) and keeps a sorted list of its k + 1 best
// columns (ranked by H, then the lower column index); the warp merges the 32
// lists with shuffles.  Rows of 512 columns or more rank quads instead, by
// their largest H (then the lower quad index), which inserts a quarter as
// often: the top k + 1 columns lie in the k + 1 best quads (a quad ranked
// before the quad of a top column holds a column ranked before that column,
// and there are fewer than k + 1 of those), so the warp evaluates the 4 (k +
// 1) columns of those quads again (the same arithmetic, bitwise the same H)
// and merges them into the row's top k + 1.  The row's kept ids and its two
// thresholds go to shared memory.  Pass 2, one thread per
// column quad: the thread walks the tile's rows in order and sums P (and the
// Switch probabilities) in registers, then writes the tile's column sums;
// route_reduce adds the tiles in a fixed order, so the load is bitwise
// reproducible.
#include <float.h>
#include <limits.h>

#include "internal.h"
#include "phi.cuh"
#include "philox.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

constexpr int NW = 8;  // warps per routing block

// H of the columns of quad m (4m .. 4m+3) of a row: c, plus the selection
// bias (sigmoid router) or eps * s (noise on); columns past nb get c = -inf.
__device__ __forceinline__ void quad_h(const RouteArgs &a, const float *crow, const float *srow,
                                       int m, int nb, bool vec4, uint32_t ctr0, uint32_t gate_id,
                                       uint32_t key0, uint32_t key1, float (&cv)[4],
                                       float (&sv)[4], float (&h)[4]) {
  const int i0 = 4 * m;
#pragma unroll
  for (int j = 0; j < 4; ++j) sv[j] = 0.f;
  if (vec4) {
    const float4 c4 = *reinterpret_cast<const float4 *>(crow + i0);
    cv[0] = c4.x; cv[1] = c4.y; cv[2] = c4.z; cv[3] = c4.w;
    if (a.noise) {
      const float4 s4 = *reinterpret_cast<const float4 *>(srow + i0);
      sv[0] = s4.x; sv[1] = s4.y; sv[2] = s4.z; sv[3] = s4.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cv[j] = i0 + j < nb ? crow[i0 + j] : -INFINITY;
      if (a.noise) sv[j] = i0 + j < nb ? srow[i0 + j] : 0.f;
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = cv[j];
  if (a.sel_bias) {  // sigmoid router: the bias enters the routing score only
    float bv[4];
    if (vec4) {
      const float4 b4 = *reinterpret_cast<const float4 *>(a.sel_bias + i0);
      bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = i0 + j < nb ? a.sel_bias[i0 + j] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) h[j] = cv[j] + bv[j];
  } else if (a.noise) {
    const uint4 wd = philox4x32_10(make_uint4(ctr0, (uint32_t)m, gate_id, 0u), key0, key1);
    float z[4];
    box_muller2(wd.x, wd.y, z[0], z[1]);
    box_muller2(wd.z, wd.w, z[2], z[3]);
#pragma unroll
    for (int j = 0; j < 4; ++j) h[j] = fmaf(z[j], sv[j], cv[j]);
  }
}

// K1 rounds of an arg-max over the heads of the sorted lists of each aligned
// group of lpr lanes (32, 16 or 8: one row each); the owner pops its head.  S
// gets the group's K1 first entries, in order.  Every lane of the warp takes
// part.
template <int K1, int LN>
__device__ __forceinline__ void warp_merge(Cand (&L)[LN], Cand (&S)[K1], int lpr) {
#pragma unroll
  for (int r = 0; r < K1; ++r) {
    float bv = L[0].v;
    int bi = L[0].i;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      if (off >= lpr) continue;
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (before(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    S[r].v = bv;
    S[r].i = bi;
    if (L[0].i == bi && bi != INT_MAX) {
#pragma unroll
      for (int j = 0; j < LN - 1; ++j) L[j] = L[j + 1];
      L[LN - 1].v = -INFINITY;
      L[LN - 1].i = INT_MAX;
    }
  }
}

// K1 = k + 1; MAXQ = column quads per thread (nb <= MAXQ * 4 * 256); SW =
// Switch router (probability sums kept).
// EX = extra outputs compiled in: the router statistics (stats_part) and the
// rows' thresholds for the backward pass (kth), each only when its pointer is
// set.
// NARROW: rows of at most 128 columns and tiles of at least 16 rows, several
// rows per warp in pass 1 (a separate instance, so that one row per warp pays
// nothing for it).
template <int K1, int MAXQ, bool SW, bool EX, bool NARROW>
__global__ void __launch_bounds__(NW * 32, (MAXQ > 4 || SW) ? 3 : 4) route_kernel(RouteArgs a) {
  constexpr int KM = K1 - 1;  // k
  constexpr int PQ = SW ? MAXQ : 1;
  // per row of a round: kept columns (one bit each, nwords words a row), the
  // (k+1)-th and k-th largest H, the Switch softmax's max and sum
  __shared__ uint32_t kept_s[NW * MAXQ * 32];
  __shared__ float thr_s[NW * 4][2];
  __shared__ float sm_s[NW * 4][2];
  __shared__ float4 red_s[NW * 32];
  __shared__ float4 redp_s[NW * 32];
  const int nb = a.nb;

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

  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = a.k;
  const bool vec4 = (nb & 3) == 0;  // rows start 16-byte aligned
  constexpr bool sw = SW;
  const uint64_t seed = a.seed_dev ? (uint64_t)__ldg(a.seed_dev) : a.seed;
  const uint32_t key0 = (uint32_t)(seed & 0xffffffffu), key1 = (uint32_t)(seed >> 32);
  const uint32_t gate_id = a.secondary ? (uint32_t)(1 + g) : 0u;
  bool bad = false;

  // pass 1: rows per warp and lanes per row; NR rows per round
  const bool by_quad = nb >= 512;  // rank quads: at least four quads per lane
  const int RPW = NARROW ? 4 : 1;
  const int LPR = 32 / RPW, sub = lane / LPR, sl = lane % LPR;
  const int NR = NW * RPW;
  // pass-2 thread layout: thread per column quad; with fewer quads than
  // threads, RG groups of threads split the rows of each round
  const int nq = (nb + 3) >> 2;
  const int RG = nq >= NW * 32 ? 1 : min((NW * 32) / nq, NR);
  const int rg = nq >= NW * 32 ? 0 : (int)threadIdx.x / nq;
  const int nqpass = (nq + NW * 32 - 1) / (NW * 32);  // quads per thread when RG == 1
  float acc[MAXQ][4], pacc[PQ][4];
#pragma unroll
  for (int u = 0; u < MAXQ; ++u)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[u][j] = 0.f;
#pragma unroll
  for (int u = 0; u < PQ; ++u)
#pragma unroll
    for (int j = 0; j < 4; ++j) pacc[u][j] = 0.f;

  const bool stats = EX && a.stats_part != nullptr;
  float rz = 0.f, rh = 0.f;  // lanes sl = 0: their rows' |c|^2 and entropies
  const int nwords = (nb + 31) >> 5;
  for (int rb = row0; rb < row_end; rb += NR) {
    // ================= pass 1: routing of row rb + rloc (LPR lanes per row)
    const int rloc = w * RPW + sub, row = rb + rloc;
    const bool live = row < row_end;
    for (int q = lane; q < RPW * nwords; q += 32) kept_s[w * RPW * nwords + q] = 0u;  // read by pass 2
    __syncwarp();
    {
      const int nbe = live ? nb : 0;  // a row past the tile's end scans nothing
      const int t = live ? (a.row_token ? a.row_token[row] : row) : 0;
      const float *crow = a.c + (size_t)(live ? row : row0) * nb;
      const float *srow = a.s + (size_t)(live ? row : row0) * nb;

      Cand L[K1];
#pragma unroll
      for (int j = 0; j < K1; ++j) { L[j].v = -INFINITY; L[j].i = INT_MAX; }
      float mx = -INFINITY, se = 0.f;  // online softmax of c (Switch)

      const uint32_t ctr0 = (uint32_t)t + a.token_base;
      for (int m = sl; 4 * m < nbe; m += LPR) {
        const int i0 = 4 * m;
        float cv[4], sv[4], h[4];
        quad_h(a, crow, srow, m, nb, vec4, ctr0, gate_id, key0, key1, cv, sv, h);
        float qm = -INFINITY;  // the quad's largest H (NaN never ranks)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (i0 + j >= nb) break;
          bad |= !isfinite(h[j]);
          if (by_quad) qm = fmaxf(qm, h[j]);
          else insert<K1>(L, h[j], i0 + j);
          if (sw) {
            const float m2 = fmaxf(mx, cv[j]);
            se = se * expf(mx - m2) + expf(cv[j] - m2);
            mx = m2;
          }
        }
        if (by_quad) insert<K1>(L, qm, m);
      }

      // the row's k + 1 best quads, then their columns again: each lane holds
      // (at most) two of the 4 (k + 1) columns, and the warp merges them
      Cand S[K1];
      if (!by_quad) {
        warp_merge<K1, K1>(L, S, LPR);
      } else {  // one row per warp here
      Cand Q[K1];
      warp_merge<K1, K1>(L, Q, 32);
      Cand C2[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) { C2[j].v = -INFINITY; C2[j].i = INT_MAX; }
#pragma unroll
      for (int l0 = 0; l0 < 4 * K1; l0 += 32) {
        const int l = l0 + lane, r = l >> 2, q = l & 3;
        int m = INT_MAX;
#pragma unroll
        for (int rr = 0; rr < K1; ++rr)
          if (rr == r) m = Q[rr].i;
        if (live && l < 4 * K1 && m != INT_MAX && 4 * m + q < nb) {
          float cv[4], sv[4], h[4];
          quad_h(a, crow, srow, m, nb, vec4, ctr0, gate_id, key0, key1, cv, sv, h);
          insert<2>(C2, q == 0 ? h[0] : q == 1 ? h[1] : q == 2 ? h[2] : h[3], 4 * m + q);
        }
      }
      warp_merge<K1, 2>(C2, S, 32);
      }

      float M = 0.f, SE = 1.f;
      if (sw) {
        M = mx; SE = se;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          if (off >= LPR) continue;
          const float om = __shfl_xor_sync(0xffffffffu, M, off);
          const float os = __shfl_xor_sync(0xffffffffu, SE, off);
          const float m2 = fmaxf(M, om);
          const float a1 = (M == -INFINITY) ? 0.f : SE * expf(M - m2);
          const float a2 = (om == -INFINITY) ? 0.f : os * expf(om - m2);
          M = m2;
          SE = a1 + a2;
        }
      }

      // gates: softmax over the kept k (Switch: the winner's full-softmax p;
      // sigmoid router: Sigmoid(c) of the kept, normalised over them)
      float gate_j = 0.f;
      int idx_j = 0;
      if (a.router == MOE_ROUTER_SIGMOID) {
        float sg[KM], den = 0.f;
#pragma unroll
        for (int j = 0; j < KM; ++j) {
          sg[j] = live && S[j].i < nb ? 1.f / (1.f + expf(-crow[S[j].i])) : 0.f;
          den += sg[j];
        }
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (j == sl) {
            idx_j = S[j].i;
            gate_j = sg[j] / den;
          }
      } else {
        float den = 0.f;
#pragma unroll
        for (int j = 0; j < KM; ++j) den += expf(S[j].v - S[0].v);
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (j == sl) {
            idx_j = S[j].i;
            gate_j = sw ? (live && S[0].i < nb ? expf(crow[S[0].i] - M) / SE : 0.f)
                        : expf(S[j].v - S[0].v) / den;
          }
      }
      if (EX && a.gate_raw && live && sl < k) {  // kept for the backward pass, by row
        a.gate_raw[(size_t)row * k + sl] = gate_j;
        a.idx_raw[(size_t)row * k + sl] = idx_j;
      }
      if (live && sl < k) {
        int slot = sl;
        float gmul = 1.f;
        int ebase = 0;
        if (a.secondary) {
          const int ps = a.row_slot[row];
          slot = ps * k + sl;
          gmul = a.gate_mult[(size_t)t * a.k1 + ps];
          ebase = g * a.expert_stride;
        }
        a.out_idx[(size_t)t * a.K + slot] = ebase + idx_j;
        a.out_gate[(size_t)t * a.K + slot] = gmul * gate_j;
      }
      if (live && sl == 0) {
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (S[j].i >= 0 && S[j].i < nb)
            kept_s[rloc * nwords + (S[j].i >> 5)] |= 1u << (S[j].i & 31);
        thr_s[rloc][0] = S[K1 - 1].v;  // -inf if the (k+1)-th does not exist
        thr_s[rloc][1] = S[K1 - 2].v;
        if (EX && a.kth)  // kept for the backward pass's load gradient
          a.kth[row] = make_int4(__float_as_int(S[K1 - 1].v), S[K1 - 1].i,
                                 __float_as_int(S[K1 - 2].v), S[K1 - 2].i);
        sm_s[rloc][0] = M;
        sm_s[rloc][1] = SE;
      }
      if (stats) {
        // router statistics of the row, a second pass over its clean logits
        // (cache hits): sum c^2 and an online softmax with S = sum e^(c-m),
        // Q = sum e^(c-m) (c-m), the entropy being log S - Q/S
        float zs = 0.f, sm = -INFINITY, ss = 0.f, sq = 0.f;
        for (int i = sl; i < nbe; i += LPR) {
          const float v = crow[i];
          zs = fmaf(v, v, zs);
          if (v > sm) {  // rescale to the new maximum
            const float r = ss > 0.f ? expf(sm - v) : 0.f;
            sq = ss > 0.f ? r * (sq + ss * (sm - v)) : 0.f;
            ss *= r;
            sm = v;
          }
          const float e = expf(v - sm);
          ss += e;
          sq = fmaf(e, v - sm, sq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          if (off >= LPR) continue;
          zs += __shfl_xor_sync(0xffffffffu, zs, off);
          const float om = __shfl_xor_sync(0xffffffffu, sm, off);
          const float os = __shfl_xor_sync(0xffffffffu, ss, off);
          const float oq = __shfl_xor_sync(0xffffffffu, sq, off);
          const float m2 = fmaxf(sm, om);
          const float r1 = ss > 0.f ? expf(sm - m2) : 0.f, r2 = os > 0.f ? expf(om - m2) : 0.f;
          sq = (ss > 0.f ? r1 * (sq + ss * (sm - m2)) : 0.f) +
               (os > 0.f ? r2 * (oq + os * (om - m2)) : 0.f);
          ss = ss * r1 + os * r2;
          sm = m2;
        }
        if (live && sl == 0) {
          rz += zs;
          rh += logf(ss) - sq / ss;
        }
      }
    }
    __syncthreads();

    // ================= pass 2: this round's rows into the column sums
    const int nrow_blk = min(NR, row_end - rb);
    if (rg < RG) {
#pragma unroll
      for (int u = 0; u < MAXQ; ++u) {
        if (u >= nqpass) break;
        const int m = (RG == 1) ? u * NW * 32 + (int)threadIdx.x : (int)threadIdx.x % nq;
        if (m >= nq) break;
        const int i0 = 4 * m;
        for (int r = rg; r < nrow_blk; r += RG) {
          const float *crow = a.c + (size_t)(rb + r) * nb;
          const float *srow = a.s + (size_t)(rb + r) * nb;
          float cv[4], sv[4] = {1.f, 1.f, 1.f, 1.f};
          if (vec4) {
            const float4 c4 = *reinterpret_cast<const float4 *>(crow + i0);
            cv[0] = c4.x; cv[1] = c4.y; cv[2] = c4.z; cv[3] = c4.w;
            if (a.noise) {
              const float4 s4 = *reinterpret_cast<const float4 *>(srow + i0);
              sv[0] = s4.x; sv[1] = s4.y; sv[2] = s4.z; sv[3] = s4.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              cv[j] = i0 + j < nb ? crow[i0 + j] : 0.f;
              if (a.noise) sv[j] = i0 + j < nb ? srow[i0 + j] : 1.f;
            }
          }
          const float thr_kept = thr_s[r][0], thr_out = thr_s[r][1];
          const uint32_t kbits = kept_s[r * nwords + (i0 >> 5)] >> (i0 & 31);  // the quad's 4 bits
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool kept = (kbits >> j) & 1u;
            float P;
            if (!a.noise) {
              P = kept ? 1.f : 0.f;
            } else {
              // thr = -inf (no (k+1)-th) gives z = +inf and P = 1; s = 0 gives
              // z = +-inf (P = 1 or 0) or, when c = thr, 0 / 0: P = 1/2
              const float thr = kept ? thr_kept : thr_out;
              const float z = __fdividef(cv[j] - thr, sv[j]);
              P = z == z ? phi_cdf(z) : 0.5f;
            }
            acc[u][j] += P;
            if (SW) pacc[u < PQ ? u : 0][j] += expf(cv[j] - sm_s[r][0]) / sm_s[r][1];
          }
        }
      }
    }
    __syncthreads();  // the next block of rows reuses kept_s / thr_s / sm_s
  }
  if (bad && a.status) atomicOr(a.status, MOE_STATUS_NONFINITE);

  if (stats) {  // the tile's statistics: a warp's rows, then warps in warp order
    __shared__ float st_s[NW][2];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {  // the row groups' leaders (other lanes hold 0)
      if (off < LPR) continue;
      rz += __shfl_xor_sync(0xffffffffu, rz, off);
      rh += __shfl_xor_sync(0xffffffffu, rh, off);
    }
    if (lane == 0) {
      st_s[w][0] = rz;
      st_s[w][1] = rh;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float z = 0.f, hh = 0.f;
#pragma unroll
      for (int q = 0; q < NW; ++q) {
        z += st_s[q][0];
        hh += st_s[q][1];
      }
      a.stats_part[(size_t)tile * 2] = z;
      a.stats_part[(size_t)tile * 2 + 1] = hh;
    }
  }

  // ---- the tile's column sums: row groups added in group order
  float *outp = a.load_part + (size_t)tile * nb;
  float *outq = sw && a.psum_part ? a.psum_part + (size_t)tile * nb : nullptr;
  auto store4 = [&](int i0, const float *v, float *dst) {
    if (vec4) {
      *reinterpret_cast<float4 *>(dst + i0) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (i0 + j < nb) dst[i0 + j] = v[j];
    }
  };
  if (RG == 1) {
#pragma unroll
    for (int u = 0; u < MAXQ; ++u) {
      if (u >= nqpass) break;
      const int m = u * NW * 32 + (int)threadIdx.x;
      if (m >= nq) break;
      store4(4 * m, acc[u], outp);
      if (SW && outq) store4(4 * m, pacc[u < PQ ? u : 0], outq);
    }
  } else {
    red_s[threadIdx.x] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
    redp_s[threadIdx.x] = make_float4(pacc[0][0], pacc[0][1], pacc[0][2], pacc[0][3]);
    __syncthreads();
    if ((int)threadIdx.x < nq) {
      float t4[4] = {0.f, 0.f, 0.f, 0.f}, p4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int q = 0; q < RG; ++q) {
        const float4 u = red_s[q * nq + threadIdx.x], v = redp_s[q * nq + threadIdx.x];
        t4[0] += u.x; t4[1] += u.y; t4[2] += u.z; t4[3] += u.w;
        p4[0] += v.x; p4[1] += v.y; p4[2] += v.z; p4[3] += v.w;
      }
      store4(4 * threadIdx.x, t4, outp);
      if (outq) store4(4 * threadIdx.x, p4, outq);
    }
  }
}

// out[g][j] = sum over the tiles of group g, in tile order within each of
// RR interleaved lanes of tiles, then the RR partial sums in fixed order:
// the same summation order on every run.
constexpr int RC = 32, RR = 32;  // columns x tile-lanes per block
__global__ void __launch_bounds__(RC * RR) route_reduce_kernel(const float *part,
                                                               const int *seg_tiles,
                                                               int ntiles_flat, int nb,
                                                               float *out) {
  __shared__ float acc[RR][RC + 1];
  const int g = blockIdx.y;
  const int j = blockIdx.x * RC + threadIdx.x;
  const int t0 = seg_tiles ? seg_tiles[g] : 0;
  const int t1 = seg_tiles ? seg_tiles[g + 1] : ntiles_flat;
  float sum = 0.f;
  if (j < nb) {
#pragma unroll 8
    for (int t = t0 + (int)threadIdx.y; t < t1; t += RR) sum += part[(size_t)t * nb + j];
  }
  acc[threadIdx.y][threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.y == 0 && j < nb) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RR; ++r) s += acc[r][threadIdx.x];
    out[(size_t)g * nb + j] = s;
  }
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
  auto go = [&](auto kern) -> int {
    return launch("route_topk", kern, dim3(tiles_upper), dim3(NW * 32), 0, st, a);
  };
  const bool wide = a.nb > 4 * 4 * NW * 32;  // more than 4096 columns
  const bool narrow = a.nb <= 128 && a.RT >= 2 * NW;
  const bool st_on = a.stats_part != nullptr || a.kth != nullptr || a.gate_raw != nullptr;
  if (a.router == MOE_ROUTER_SWITCH) {
    if (a.k != 1 || wide) return MOE_EINVAL;
    if (narrow)
      return st_on ? go(route_kernel<2, 4, true, true, true>) : go(route_kernel<2, 4, true, false, true>);
    return st_on ? go(route_kernel<2, 4, true, true, false>) : go(route_kernel<2, 4, true, false, false>);
  }
#define MOE_ROUTE_CASE(K1)                                                               \
  case K1:                                                                               \
    if (narrow)                                                                          \
      return st_on ? go(route_kernel<K1, 4, false, true, true>)                          \
                   : go(route_kernel<K1, 4, false, false, true>);                        \
    if (st_on)                                                                           \
      return wide ? go(route_kernel<K1, 8, false, true, false>)                          \
                  : go(route_kernel<K1, 4, false, true, false>);                         \
    return wide ? go(route_kernel<K1, 8, false, false, false>)                           \
                : go(route_kernel<K1, 4, false, false, false>);
  switch (a.k + 1) {
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(3)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(5)
    MOE_ROUTE_CASE(6)
    MOE_ROUTE_CASE(7)
    MOE_ROUTE_CASE(8)
    MOE_ROUTE_CASE(9)
    default: return MOE_EINVAL;
  }
#undef MOE_ROUTE_CASE
}

int launch_route_reduce(const float *part, const int *seg_tiles, int G, int ntiles_flat, int nb,
                        float *out, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(nb, RC), G);
  return launch("route_reduce", route_reduce_kernel, grid, dim3(RC, RR), 0, st, part, seg_tiles,
                ntiles_flat, nb, out);
}

int launch_hier_load(const float *load_p, const float *load2, const int *cnt, int a, int b,
                     float *load, cudaStream_t st) {
  return launch("hier_load", hier_load_kernel, dim3((unsigned)ceil_div((int64_t)a * b, 256)),
                dim3(256), 0, st, load_p, load2, cnt, a, b, load);
}

}  // namespace moe
