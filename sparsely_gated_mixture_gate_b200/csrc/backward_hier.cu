// backward_hier.cu -- the gate side of the hierarchical layer's backward pass.
//
// [SGMoE-note] "分层 MoE": token t's slot ps*k2+ss is expert g*b + j, g the
// ps-th kept group of the primary gate and j the ss-th kept expert of g's
// gate, with gate G_p(x)_g * G_g(x)_j.  The pages give no backward formulas;
// the loss is the forward's (upstream gradient times y plus the weighted
// balancing losses), with the hierarchical Load read as Load(g*b+j) =
// Load_p(X)_g * Load_g(X_g)_j / |X_g| (|X_g| a count, no gradient).  So:
//   slot gradient dS = dL/dgate + dL/dImportance(e)       (hier_split)
//   dL/dG_p(g) = sum_ss dS * G_g(j),  dL/dG_g(j) = dS * G_p(g)
//   load coefficients: lam_p(g) = sum_j lamL(g*b+j) Load_g_j / |X_g|,
//                      lam_s(g, j) = lamL(g*b+j) Load_p_g / |X_g|  (hier_coef)
// after which each level is a flat noisy top-k gate (gate_bwd, with the
// secondary rows' tokens, noise streams 1 + g and coefficients lam_s(g, .)),
// and the secondary gates' projections, one per group and gathered rows,
// take these contractions (fp32, every output summed by one thread in row
// order, so the results are bitwise reproducible):
//   dW_g2[g] = sum over g's rows r of x[token(r)] (x) dc2[r]   (and dW_noise2)
//   db_g2[g] = sum over g's rows of dc2[r]
//   dx[t]   += sum_ps (dc2[r] W_g2[g]^T + dz2[r] W_noise2[g]^T), r = row of (t, ps)
#include <algorithm>

#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

// one block per group; lam_p by a fixed-order block sum
__global__ void __launch_bounds__(NT) hier_coef_kernel(const float *lam_load, const float *load_p,
                                                       const float *load2, const int *cnt, int b,
                                                       float *lam_p, float *lam_s) {
  __shared__ float part[NT / 32];
  const int g = blockIdx.x;
  const int c = cnt[g];
  const float inv = c > 0 ? 1.f / (float)c : 0.f;
  float acc = 0.f;
  for (int j = threadIdx.x; j < b; j += NT) {
    const float l = lam_load[(size_t)g * b + j];
    lam_s[(size_t)g * b + j] = c > 0 ? l * load_p[g] * inv : 0.f;
    acc = fmaf(l, load2[(size_t)g * b + j] * inv, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += part[w];
    lam_p[g] = c > 0 ? s : 0.f;
  }
}

// one thread per (token, kept group)
__global__ void hier_split_kernel(int T, int k1, int k2, int K, int n, const float *pgate,
                                  const int *grow, const int *topk_idx, const float *dgate,
                                  const float *gate2, const float *lam_imp, float *dgp,
                                  float *dgs) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= T * k1) return;
  const int t = u / k1, ps = u % k1;
  const float Gp = pgate[u];
  const int r = grow[u];
  if (r < 0 || r >= T * k1) {  // an unplaced pair: only after non-finite logits
    dgp[u] = 0.f;
    return;
  }
  float acc = 0.f;
  for (int ss = 0; ss < k2; ++ss) {
    const size_t slot = (size_t)t * K + (size_t)ps * k2 + ss;
    const int e = topk_idx[slot];  // out of range only after non-finite logits
    const float dS = dgate[slot] + (e >= 0 && e < n ? lam_imp[e] : 0.f);
    acc = fmaf(dS, gate2[(size_t)r * k2 + ss], acc);
    dgs[(size_t)r * k2 + ss] = dS * Gp;
  }
  dgp[u] = acc;
}

// dW[g] [d][b] = sum over the group's rows of x[token(r)] (x) D[r]; blockIdx.z
// picks the projection (0: dc2 -> dW_g2, 1: dz2 -> dW_noise2)
constexpr int WT = 64, WR = 32;
__global__ void __launch_bounds__(NT) hier_wgrad_kernel(const float *__restrict__ x, int d,
                                                        const int *__restrict__ row_token,
                                                        const int *__restrict__ seg_off, int b,
                                                        const float *__restrict__ D0,
                                                        const float *__restrict__ D1, float *dW0,
                                                        float *dW1) {
  __shared__ float Xs[WR][WT + 4];
  __shared__ float Ds[WR][WT + 4];
  const int g = blockIdx.x, q0 = blockIdx.y * WT, j0 = blockIdx.z % ((b + WT - 1) / WT) * WT;
  const int proj = blockIdx.z / ((b + WT - 1) / WT);
  const float *D = proj ? D1 : D0;
  float *dW = (proj ? dW1 : dW0) + (size_t)g * d * b;
  const int r_beg = seg_off[g], r_end = seg_off[g + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int r0 = r_beg; r0 < r_end; r0 += WR) {
    for (int e = threadIdx.x; e < WR * WT; e += NT) {
      const int rr = e / WT, cc = e % WT, r = r0 + rr;
      const bool ok = r < r_end;
      Xs[rr][cc] = ok && q0 + cc < d ? __ldg(x + (size_t)row_token[r] * d + q0 + cc) : 0.f;
      Ds[rr][cc] = ok && j0 + cc < b ? __ldg(D + (size_t)r * b + j0 + cc) : 0.f;
    }
    __syncthreads();
    const int nr = min(WR, r_end - r0);
    for (int rr = 0; rr < nr; ++rr) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(Xs[rr][ty * 4 + i], Ds[rr][tx * 4 + j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = q0 + ty * 4 + i;
    if (q >= d) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int jj = j0 + tx * 4 + j;
      if (jj < b) dW[(size_t)q * b + jj] = acc[i][j];
    }
  }
}

// db[g][j] = sum over the group's rows of D[r][j], rows in order
__global__ void hier_colsum_kernel(const int *seg_off, int b, const float *D, float *db) {
  const int g = blockIdx.x, j = blockIdx.y * blockDim.x + threadIdx.x;
  if (j >= b) return;
  float s = 0.f;
  for (int r = seg_off[g]; r < seg_off[g + 1]; ++r) s += D[(size_t)r * b + j];
  db[(size_t)g * b + j] = s;
}

// dxs[r][q] = sum_j dc2[r][j] W_g2[g][q][j] + sum_j dz2[r][j] W_noise2[g][q][j]
// over 128-row tiles of one group (seg_mblk: the groups' tile prefix)
constexpr int DM = kGateBM, DQ = 64, DK = 16;  // the groups' 128-row tiles (seg_mblk)
__global__ void __launch_bounds__(NT) hier_dgrad_kernel(const float *__restrict__ dc2,
                                                        const float *__restrict__ dz2,
                                                        const float *__restrict__ Wg2,
                                                        const float *__restrict__ Wn2,
                                                        const int *seg_off, const int *seg_mblk,
                                                        int G, int d, int b, float *dxs) {
  __shared__ float Dsh[DM][DK + 1];
  __shared__ float Wsh[DK][DQ + 4];
  const int mblk = blockIdx.x;
  if (mblk >= seg_mblk[G]) return;
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seg_mblk[mid] <= mblk) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int row0 = seg_off[g] + (mblk - seg_mblk[g]) * DM, row_end = seg_off[g + 1];
  const int q0 = blockIdx.y * DQ;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int proj = 0; proj < (dz2 ? 2 : 1); ++proj) {
    const float *D = proj ? dz2 : dc2;
    const float *W = (proj ? Wn2 : Wg2) + (size_t)g * d * b;
    for (int j0 = 0; j0 < b; j0 += DK) {
      for (int e = threadIdx.x; e < DM * DK; e += NT) {
        const int rr = e / DK, kk = e % DK, r = row0 + rr;
        Dsh[rr][kk] = r < row_end && j0 + kk < b ? __ldg(D + (size_t)r * b + j0 + kk) : 0.f;
      }
      for (int e = threadIdx.x; e < DK * DQ; e += NT) {
        const int qq = e / DK, kk = e % DK;
        Wsh[kk][qq] = q0 + qq < d && j0 + kk < b ? __ldg(W + (size_t)(q0 + qq) * b + j0 + kk) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < DK; ++kk)
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(Dsh[ty * 8 + i][kk], Wsh[kk][tx * 4 + j], acc[i][j]);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = row0 + ty * 8 + i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = q0 + tx * 4 + j;
      if (q < d) dxs[(size_t)r * d + q] = acc[i][j];
    }
  }
}

// dx[t][q] += sum over the kept groups ps of dxs[row of (t, ps)][q], ps in order
__global__ void hier_dx_sum_kernel(int T, int k1, int d, const int *grow, const float *dxs,
                                   float *dx) {
  const int64_t total = (int64_t)T * d;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(e / d), q = (int)(e % d);
    float s = dx[e];
    for (int ps = 0; ps < k1; ++ps) {
      const int r = grow[(size_t)t * k1 + ps];  // -1: unplaced (non-finite logits)
      if (r >= 0 && r < T * k1) s += dxs[(size_t)r * d + q];
    }
    dx[e] = s;
  }
}

}  // namespace

int launch_hier_coef(const float *lam_load, const float *load_p, const float *load2,
                     const int *cnt, int a, int b, float *lam_p, float *lam_s, cudaStream_t st) {
  return launch("hier_coef", hier_coef_kernel, dim3((unsigned)a), dim3(NT), 0, st, lam_load, load_p,
                load2, cnt, b, lam_p, lam_s);
}

int launch_hier_split(int T, int k1, int k2, int K, int n, const float *pgate,
                      const int *grow, const int *topk_idx, const float *dgate,
                      const float *gate2, const float *lam_imp, float *dgp, float *dgs,
                      cudaStream_t st) {
  const int64_t u = (int64_t)T * k1;
  return launch("hier_split", hier_split_kernel, dim3((unsigned)ceil_div(u, NT)), dim3(NT), 0, st, T,
                k1, k2, K, n, pgate, grow, topk_idx, dgate, gate2, lam_imp, dgp, dgs);
}

int launch_hier_gate_wgrad(const float *x, int d, const int *row_token, const int *seg_off, int a,
                           int b, const float *dc2, const float *dz2, float *dWg2, float *dWn2,
                           float *dbg2, cudaStream_t st) {
  const int nj = (int)ceil_div(b, WT);
  if (dWg2 || dWn2) {
    // both projections in one launch when both are asked for
    const bool two = dWg2 && dWn2 && dz2;
    const float *D0 = dWg2 ? dc2 : dz2;
    float *W0 = dWg2 ? dWg2 : dWn2;
    MOE_TRY(launch("hier_gate_wgrad", hier_wgrad_kernel,
                   dim3((unsigned)a, (unsigned)ceil_div(d, WT), (unsigned)(nj * (two ? 2 : 1))),
                   dim3(NT), 0, st, x, d, row_token, seg_off, b, D0, two ? dz2 : D0, W0,
                   two ? dWn2 : W0));
  }
  if (dbg2)
    MOE_TRY(launch("hier_colsum", hier_colsum_kernel, dim3((unsigned)a, (unsigned)ceil_div(b, NT)),
                   dim3(NT), 0, st, seg_off, b, dc2, dbg2));
  return MOE_OK;
}

int launch_hier_gate_dgrad(const float *dc2, const float *dz2, const float *Wg2, const float *Wn2,
                           const int *seg_off, const int *seg_mblk, int mblk_upper, int a, int d,
                           int b, float *dxs, int T, int k1, const int *grow, float *dx,
                           cudaStream_t st) {
  MOE_TRY(launch("hier_gate_dgrad", hier_dgrad_kernel,
                 dim3((unsigned)mblk_upper, (unsigned)ceil_div(d, DQ)), dim3(NT), 0, st, dc2, dz2,
                 Wg2, Wn2, seg_off, seg_mblk, a, d, b, dxs));
  const int64_t total = (int64_t)T * d;
  const int grid = (int)std::min<int64_t>(ceil_div(total, NT), 8 * (int64_t)num_sms());
  return launch("hier_dx_sum", hier_dx_sum_kernel, dim3((unsigned)(grid > 0 ? grid : 1)), dim3(NT),
                0, st, T, k1, d, grow, dxs, dx);
}

}  // namespace moe
