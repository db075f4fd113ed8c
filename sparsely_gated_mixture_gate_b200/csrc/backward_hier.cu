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
// take these contractions (fp32; grad_gemm.cu's kernel in its grouped mode,
// every output one fused multiply-add chain in row or column order, so the
// results are bitwise reproducible):
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

// db[g][j] = sum over the group's rows of D[r][j]: 8 row lanes per column
// (lane l adds rows l, l + 8, ... in order), then the lanes in order
constexpr int CL = 8, CC = 32;  // row lanes x columns per block
__global__ void __launch_bounds__(CL * CC) hier_colsum_kernel(const int *seg_off, int b,
                                                              const float *D, float *db) {
  __shared__ float part[CL][CC + 1];
  const int g = blockIdx.x, c = threadIdx.x % CC, l = threadIdx.x / CC;
  const int j = blockIdx.y * CC + c;
  const int r0 = seg_off[g], r1 = seg_off[g + 1];
  float s = 0.f;
  if (j < b)
    for (int r = r0 + l; r < r1; r += CL) s += __ldg(D + (size_t)r * b + j);
  part[l][c] = s;
  __syncthreads();
  if (l == 0 && j < b) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < CL; ++q) t += part[q][c];
    db[(size_t)g * b + j] = t;
  }
}

// dx[t][q] += sum over the kept groups ps of dxs[row of (t, ps)][q], ps in
// order; four columns per thread (d is a multiple of 8)
__global__ void hier_dx_sum_kernel(int T, int k1, int d, const int *grow, const float *dxs,
                                   float *dx) {
  const int d4 = d >> 2;
  const int64_t total = (int64_t)T * d4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(e / d4), q4 = (int)(e % d4);
    float4 s = reinterpret_cast<float4 *>(dx)[e];
    for (int ps = 0; ps < k1; ++ps) {
      const int r = grow[(size_t)t * k1 + ps];  // -1: unplaced (non-finite logits)
      if (r >= 0 && r < T * k1) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(dxs + (size_t)r * d) + q4);
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
    }
    reinterpret_cast<float4 *>(dx)[e] = s;
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
  if (dWg2 || dWn2) {
    // dW[g] = X_g^T D_g: M = d, N = b, K = the group's rows (x rows gathered
    // by token); both projections in one launch when both are asked for
    SgemmArgs s{};
    s.M = d;
    s.N = b;
    s.K = 0;
    s.A[0] = s.A[1] = x;
    s.lda = d;
    s.at = 1;
    s.ldb = b;
    s.bt = 0;
    s.ldc = b;
    const bool two = dWg2 && dWn2 && dz2;
    s.B[0] = dWg2 ? dc2 : dz2;
    s.C[0] = dWg2 ? dWg2 : dWn2;
    s.B[1] = two ? dz2 : s.B[0];
    s.C[1] = two ? dWn2 : s.C[0];
    s.nprob = two ? 2 : 1;
    s.splits = 1;
    s.seg_off = seg_off;
    s.a_row = row_token;
    s.G = a;
    s.seg_k = 1;
    s.sC = (int64_t)d * b;
    s.name = "hier_gate_wgrad";
    MOE_TRY(launch_sgemm(s, st));
  }
  if (dbg2)
    MOE_TRY(launch("hier_colsum", hier_colsum_kernel, dim3((unsigned)a, (unsigned)ceil_div(b, CC)),
                   dim3(CL * CC), 0, st, seg_off, b, dc2, dbg2));
  return MOE_OK;
}

int launch_hier_gate_dgrad(const float *dc2, const float *dz2, const float *Wg2, const float *Wn2,
                           const int *seg_off, const int *seg_mblk, int mblk_upper, int a, int d,
                           int b, float *dxs, int T, int k1, const int *grow, float *dx,
                           cudaStream_t st) {
  // dxs[rows of g] = dc2 W_g2[g]^T (+ dz2 W_noise2[g]^T): M = the group's rows,
  // N = d, K = b; B(k, n) = W[g][n][k]
  SgemmArgs s{};
  s.M = T * k1;
  s.N = d;
  s.K = b;
  s.A[0] = dc2;
  s.A[1] = dz2;
  s.lda = b;
  s.at = 0;
  s.B[0] = Wg2;
  s.B[1] = Wn2;
  s.ldb = b;
  s.bt = 1;
  s.C[0] = s.C[1] = dxs;
  s.ldc = d;
  s.nprob = 1;
  s.ksum = dz2 ? 1 : 0;
  s.splits = 1;
  s.seg_off = seg_off;
  s.seg_mblk = seg_mblk;
  s.G = a;
  s.seg_k = 0;
  s.mblk_upper = mblk_upper;
  s.sB = (int64_t)d * b;
  s.name = "hier_gate_dgrad";
  MOE_TRY(launch_sgemm(s, st));
  const int64_t total = (int64_t)T * (d / 4);
  const int grid = (int)std::min<int64_t>(ceil_div(total, NT), 8 * (int64_t)num_sms());
  return launch("hier_dx_sum", hier_dx_sum_kernel, dim3((unsigned)(grid > 0 ? grid : 1)), dim3(NT),
                0, st, T, k1, d, grow, dxs, dx);
}

}  // namespace moe
