// backward.cu -- the layer's backward pass apart from the tensor-core GEMMs
// (expert_tc.cu, wgrad_tc.cu) and the gate's fp32 GEMMs (grad_gemm.cu).
//
// The pages give no backward formulas; they say which paths carry a
// gradient: the kept gates are smooth in the logits ([SGMoE-xyz] 常見問題),
// KeepTopK gives the experts it drops none ([SGMoE-note] 缺点与局限性), and
// the noise lets the load loss reach the gate through Phi ([SGMoE-note]
// Noisy Top-K Gating).  What follows is the chain rule of the forward pass in
// reverse order, for the loss
//   L = sum(dy * y) + w_importance CV(Importance)^2 + w_load CV(Load)^2
//       + alpha * N sum_i f_i P_i (Switch)
//   bwd_coef        dL/dImportance_i, dL/dLoad_i (through CV^2) and the Switch
//                   loss's dL/dp_ti (one block, fp64)
//   combine_bwd     per token and kept slot: dy_perm[row] = bf16(g * dy_t),
//                   dgate = <dy_t, y_perm[row]>; the shared expert's rows get dy
//   bias_grad       db of every expert: column sums of its rows of dy_perm and
//                   dhid, in a fixed order
//   expert_bwd_f32  fp32 experts: block per expert over its rows, the hidden
//                   layer recomputed, dW1, dW2, db1, db2 accumulated in place
//   dx_gather       dx_t = sum over kept slots of dx_perm[row] (+ dy_t for a
//                   passed-through token, + the shared expert's row)
//   gate_bwd        per token: dL/dc (clean logits) and dL/dz (noise logits,
//                   z = x W_noise) through the softmax over the kept, the
//                   importance and load losses (Phi' and kth_excluding), the
//                   noise (eps recomputed from Philox) and Softplus; for the
//                   noisy gate up to 1024 experts the row sits in registers
//   gate_stats_bwd  the router z-loss and gate entropy terms added to dL/dc
//   colsum          column sums of a row-major matrix in row blocks (db_g)
#include "internal.h"
#include "philox.cuh"

namespace moe {
namespace {

constexpr int CT = 256;

__device__ double block_sum_d(double v, double *sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) sh[w] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = 0.0;
    for (int i = 0; i < CT / 32; ++i) r += sh[i];
    sh[CT / 32] = r;
  }
  __syncthreads();
  const double r = sh[CT / 32];
  __syncthreads();
  return r;
}

// d CV(v)^2 / d v_i = 2 / (n mean^2) * ((v_i - mean) - var / mean), times w
// (0 where the mean is 0, as CV^2 is defined 0 there)
__device__ void cv2_grad(const float *v, int n, float w, float *out, double *sh) {
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += CT) s += (double)v[i];
  const double mean = block_sum_d(s, sh) / (double)n;
  double q = 0.0;
  for (int i = threadIdx.x; i < n; i += CT) {
    const double dv = (double)v[i] - mean;
    q += dv * dv;
  }
  const double var = block_sum_d(q, sh) / (double)n;
  for (int i = threadIdx.x; i < n; i += CT) {
    double g = 0.0;
    if (mean != 0.0 && w != 0.f)
      g = (double)w * 2.0 / ((double)n * mean * mean) * (((double)v[i] - mean) - var / mean);
    out[i] = (float)g;
  }
}

__global__ void __launch_bounds__(CT) bwd_coef_kernel(const float *importance, const float *load,
                                                      const int *counts, int n, int T, float w_imp,
                                                      float w_load, float alpha, int router,
                                                      int noise, float *lam_imp, float *lam_load,
                                                      float *sw_coef) {
  __shared__ double sh[CT / 32 + 1];
  cv2_grad(importance, n, w_imp, lam_imp, sh);
  // without noise Load is the count of selections: no gradient
  cv2_grad(load, n, noise ? w_load : 0.f, lam_load, sh);
  for (int i = threadIdx.x; i < n; i += CT) {
    // Switch: alpha N sum_i f_i P_i, P_i = sum_t p_ti / T, f_i fixed
    const double c = router == MOE_ROUTER_SWITCH && T > 0
                         ? (double)alpha * (double)n * ((double)counts[i] / (double)T) / (double)T
                         : 0.0;
    sw_coef[i] = (float)c;
  }
}

// ---------------------------------------------------------------- combine_bwd
constexpr int NT = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 pk, float (&f)[8]) {
  const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[u]));
    f[2 * u] = f2.x;
    f[2 * u + 1] = f2.y;
  }
}
__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * u], f[2 * u + 1]);
    w[u] = *reinterpret_cast<uint32_t *>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// expert rows: 8 features as bf16 (16 bytes) or fp32 (32 bytes)
template <bool BF16>
__device__ __forceinline__ void load8(const void *base, size_t row, int d, int c, float (&f)[8]) {
  if (BF16) {
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) +
                                                         row * d) + c), f);
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + row * d);
    const float4 u = __ldg(p + 2 * c), v = __ldg(p + 2 * c + 1);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
    f[4] = v.x; f[5] = v.y; f[6] = v.z; f[7] = v.w;
  }
}
template <bool BF16>
__device__ __forceinline__ void store8(void *base, size_t row, int d, int c, const float (&f)[8]) {
  if (BF16) {
    reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(base) + row * d)[c] = f32x8_to_bf16(f);
  } else {
    float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(base) + row * d);
    p[2 * c] = make_float4(f[0], f[1], f[2], f[3]);
    p[2 * c + 1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// one warp per token, 8 features per lane per step; BF16: the experts' rows
// are bf16 (the gradient reaching them is rounded to bf16 like their
// activations), else fp32
template <int KM, bool BF16>
__global__ void __launch_bounds__(NT) combine_bwd_kernel(
    const float *__restrict__ dy, const float *__restrict__ gate, const int *__restrict__ row_of,
    const void *__restrict__ y_perm, int T, int k, int d, void *__restrict__ dy_perm,
    float *__restrict__ dgate, void *__restrict__ dy_shared) {
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int rows[KM];
  float g[KM], acc[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    rows[j] = j < k ? __ldg(row_of + (size_t)t * k + j) : -1;
    g[j] = j < k ? __ldg(gate + (size_t)t * k + j) : 0.f;
    acc[j] = 0.f;
  }
  const float4 *dyr = reinterpret_cast<const float4 *>(dy + (size_t)t * d);
  for (int c = lane; c < (d >> 3); c += 32) {
    float v[8];
    {
      const float4 u = __ldg(dyr + 2 * c), w = __ldg(dyr + 2 * c + 1);
      v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
      v[4] = w.x; v[5] = w.y; v[6] = w.z; v[7] = w.w;
    }
    if (dy_shared) store8<BF16>(dy_shared, (size_t)t, d, c, v);
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (rows[j] < 0) continue;
      float yv[8], o[8];
      load8<BF16>(y_perm, (size_t)rows[j], d, c, yv);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc[j] = fmaf(v[u], yv[u], acc[j]);
        o[u] = g[j] * v[u];
      }
      store8<BF16>(dy_perm, (size_t)rows[j], d, c, o);
    }
  }
#pragma unroll
  for (int j = 0; j < KM; ++j) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
  }
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k) dgate[(size_t)t * k + j] = acc[j];  // 0 for a dropped slot
}

// ---------------------------------------------------------------- dx_gather
template <int KM, bool BF16>
__global__ void __launch_bounds__(NT) dx_gather_kernel(
    const void *__restrict__ dx_perm, const int *__restrict__ row_of,
    const float *__restrict__ dy, int passthrough, int T, int k, int d,
    const void *__restrict__ dx_shared, float *__restrict__ dx) {
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int rows[KM];
  bool any = false;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    rows[j] = j < k ? __ldg(row_of + (size_t)t * k + j) : -1;
    any |= rows[j] >= 0;
  }
  const bool pass = passthrough && !any;
  float4 *out = reinterpret_cast<float4 *>(dx + (size_t)t * d);
  for (int c = lane; c < (d >> 3); c += 32) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (rows[j] < 0) continue;
      float v[8];
      load8<BF16>(dx_perm, (size_t)rows[j], d, c, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] += v[u];
    }
    if (pass) {  // y = x for a token whose every slot overflowed
      const float4 *dyr = reinterpret_cast<const float4 *>(dy + (size_t)t * d);
      const float4 u = __ldg(dyr + 2 * c), w = __ldg(dyr + 2 * c + 1);
      a[0] += u.x; a[1] += u.y; a[2] += u.z; a[3] += u.w;
      a[4] += w.x; a[5] += w.y; a[6] += w.z; a[7] += w.w;
    }
    if (dx_shared) {
      float v[8];
      load8<BF16>(dx_shared, (size_t)t, d, c, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] += v[u];
    }
    out[2 * c] = make_float4(a[0], a[1], a[2], a[3]);
    out[2 * c + 1] = make_float4(a[4], a[5], a[6], a[7]);
  }
}

// ---------------------------------------------------------------- bias_grad
// grid.y: expert; grid.x: 256-column blocks of dy_perm (N = d) then of dhid
// (N = f).  Thread (row group rg of 8, column group cg of 32) sums 8 columns
// over rows rg, rg+8, ...; the 8 row groups are then added in order.
__global__ void __launch_bounds__(256) bias_grad_kernel(
    const __nv_bfloat16 *__restrict__ dy_perm, const __nv_bfloat16 *__restrict__ dhid,
    const int *__restrict__ offsets, int d, int f, float *__restrict__ db2,
    float *__restrict__ db1) {
  __shared__ float part[8][256];
  const int e = blockIdx.y;
  const int cb2 = (d + 255) / 256;
  const bool first = (int)blockIdx.x < cb2;
  const int N = first ? d : f;
  const int cb = first ? blockIdx.x : blockIdx.x - cb2;
  const __nv_bfloat16 *src = first ? dy_perm : dhid;
  float *const dsel = first ? db2 : db1;
  if (!dsel) return;  // that bias gradient is not wanted
  float *dst = dsel + (size_t)e * N;
  const int cg = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int c0 = cb * 256 + cg * 8;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (c0 < N) {
#pragma unroll 4
    for (int r = r0 + rg; r < r1; r += 8) {
      float v[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(src + (size_t)r * N + c0)), v);
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] += v[u];
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) part[rg][cg * 8 + u] = a[u];
  __syncthreads();
  const int col = cb * 256 + threadIdx.x;
  if (col < N) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += part[q][threadIdx.x];
    dst[col] = s;
  }
}

// ---------------------------------------------------------------- expert_bwd_f32
// fp32 experts: one block per expert walks the expert's rows in order.  Per
// row it recomputes the hidden layer exactly as the forward's fp32 kernel
// does (warp per unit, lanes over the input, the same shuffle reduction), then
//   dh = (W2^T dy_perm) * [h > 0],  dx_perm = W1^T dh,
//   dW2 += dy_perm h^T, dW1 += dh x^T, db2 += dy_perm, db1 += dh,
// accumulated in place: the block owns its expert's gradients (each element
// always updated by the same thread), so the result does not depend on timing.
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__global__ void __launch_bounds__(256) expert_bwd_f32_kernel(
    const float *__restrict__ x_perm, const float *__restrict__ dy_perm,
    const int *__restrict__ offsets, int d, int f, const float *__restrict__ W1,
    const float *__restrict__ b1, const float *__restrict__ W2, float *__restrict__ dx_perm,
    float *__restrict__ dW1, float *__restrict__ db1, float *__restrict__ dW2,
    float *__restrict__ db2) {
  extern __shared__ float sh[];
  float *xs = sh, *gs = sh + d, *hs = sh + 2 * d, *dh = sh + 2 * d + f;
  const int e = blockIdx.x, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  constexpr int NTB = 256, NWB = NTB / 32;
  const float *W1e = W1 + (size_t)e * f * d, *W2e = W2 + (size_t)e * d * f;
  float *dW1e = dW1 + (size_t)e * f * d, *dW2e = dW2 + (size_t)e * d * f;
  float *db1e = db1 ? db1 + (size_t)e * f : nullptr, *db2e = db2 ? db2 + (size_t)e * d : nullptr;
  for (int i = tid; i < f * d; i += NTB) {
    dW1e[i] = 0.f;
    dW2e[i] = 0.f;
  }
  for (int j = tid; j < f; j += NTB)
    if (db1e) db1e[j] = 0.f;
  for (int q = tid; q < d; q += NTB)
    if (db2e) db2e[q] = 0.f;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  for (int r = r0; r < r1; ++r) {
    for (int q = tid; q < d; q += NTB) {
      xs[q] = x_perm[(size_t)r * d + q];
      gs[q] = dy_perm[(size_t)r * d + q];
    }
    __syncthreads();
    for (int j = w; j < f; j += NWB) {  // the forward's hidden unit j
      const float *wr = W1e + (size_t)j * d;
      float acc = 0.f;
      for (int q = lane; q < d; q += 32) acc = fmaf(xs[q], wr[q], acc);
      acc = warp_sum_f(acc);
      if (lane == 0) hs[j] = fmaxf(acc + (b1 ? b1[(size_t)e * f + j] : 0.f), 0.f);
    }
    __syncthreads();
    for (int j = tid; j < f; j += NTB) {
      float acc = 0.f;
      for (int q = 0; q < d; ++q) acc = fmaf(W2e[(size_t)q * f + j], gs[q], acc);
      dh[j] = hs[j] > 0.f ? acc : 0.f;  // ReLU passes the gradient where it is positive
    }
    __syncthreads();
    for (int q = tid; q < d; q += NTB) {
      float acc = 0.f;
      for (int j = 0; j < f; ++j) acc = fmaf(W1e[(size_t)j * d + q], dh[j], acc);
      dx_perm[(size_t)r * d + q] = acc;
    }
    for (int i = tid; i < d * f; i += NTB) dW2e[i] = fmaf(gs[i / f], hs[i % f], dW2e[i]);
    for (int i = tid; i < f * d; i += NTB) dW1e[i] = fmaf(dh[i / d], xs[i % d], dW1e[i]);
    if (db2e)
      for (int q = tid; q < d; q += NTB) db2e[q] += gs[q];
    if (db1e)
      for (int j = tid; j < f; j += NTB) db1e[j] += dh[j];
    __syncthreads();  // xs, gs, hs, dh are rewritten by the next row
  }
}

// ---------------------------------------------------------------- gate_bwd
constexpr int GW = 8;  // warps (rows) per block

// one warp per token row of the flat gate
// the row's token (noise counter), its noise stream and its load coefficients:
// token rows use gate id 0; a secondary gate's row uses 1 + its group
struct RowCtx {
  uint32_t tok, gate_id;
  const float *lam_load;
};
__device__ __forceinline__ RowCtx row_ctx(const GateBwdArgs &a, int t) {
  RowCtx r{(uint32_t)(a.row_token ? a.row_token[t] : t) + a.token_base, 0u, a.lam_load};
  if (a.seg_off) {
    int lo = 0, hi = a.G - 1;  // largest g with seg_off[g] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.seg_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    r.gate_id = 1u + (uint32_t)lo;
    r.lam_load = a.lam_load ? a.lam_load + (size_t)lo * a.n : nullptr;
  }
  return r;
}

template <int KM>
__global__ void __launch_bounds__(GW * 32) gate_bwd_kernel(GateBwdArgs a) {
  const int t = blockIdx.x * GW + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int lane = threadIdx.x & 31;
  const int n = a.n, k = a.k;
  const RowCtx rc = row_ctx(a, t);
  const float *crow = a.c + (size_t)t * n;
  const float *srow = a.s + (size_t)t * n;
  float *dcrow = a.dc + (size_t)t * n;
  float *dzrow = a.dz ? a.dz + (size_t)t * n : nullptr;

  // the kept slots, larger H first (every lane holds all of them)
  int ids[KM];
  float gs[KM], dG[KM];
  {
    int id = 0;
    float gv = 0.f, dv = 0.f;
    if (lane < k) {
      id = a.idx[(size_t)t * k + lane];
      gv = a.gate[(size_t)t * k + lane];
      // + the importance term (an id out of range, only after non-finite
      // logits, which the forward reports, reads nothing)
      dv = a.dgate[(size_t)t * k + lane] + (a.lam_imp && id >= 0 && id < n ? a.lam_imp[id] : 0.f);
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      ids[j] = __shfl_sync(0xffffffffu, id, j);
      gs[j] = __shfl_sync(0xffffffffu, gv, j);
      dG[j] = __shfl_sync(0xffffffffu, dv, j);
    }
  }
  float gdg = 0.f;  // sum_j g_j dG_j
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j < k) gdg = fmaf(gs[j], dG[j], gdg);

  if (a.router == MOE_ROUTER_SWITCH) {
    // gate = p_argmax, p = softmax(c): dp_i = sw_i + [i = e_0] dG_0,
    // dc_i = p_i (dp_i - sum_l p_l dp_l)
    float mx = -INFINITY, se = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float v = crow[i];
      const float m2 = fmaxf(mx, v);
      se = se * expf(mx - m2) + expf(v - m2);
      mx = m2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, mx, off);
      const float os = __shfl_xor_sync(0xffffffffu, se, off);
      const float m2 = fmaxf(mx, om);
      const float a1 = mx == -INFINITY ? 0.f : se * expf(mx - m2);
      const float a2 = om == -INFINITY ? 0.f : os * expf(om - m2);
      mx = m2;
      se = a1 + a2;
    }
    float pd = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float p = expf(crow[i] - mx) / se;
      pd = fmaf(p, a.sw_coef[i] + (i == ids[0] ? dG[0] : 0.f), pd);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) pd += __shfl_xor_sync(0xffffffffu, pd, off);
    for (int i = lane; i < n; i += 32) {
      const float p = expf(crow[i] - mx) / se;
      dcrow[i] = p * (a.sw_coef[i] + (i == ids[0] ? dG[0] : 0.f) - pd);
    }
    return;
  }

  if (a.router == MOE_ROUTER_SIGMOID) {
    // g_j = sigma(c_j) / S over the kept: dc_m = (dG_m - sum g dG) / S sigma_m (1 - sigma_m)
    float sg[KM], S = 0.f;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      sg[j] = j < k ? 1.f / (1.f + expf(-crow[ids[j]])) : 0.f;
      S += sg[j];
    }
    for (int i = lane; i < n; i += 32) {
      float v = 0.f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k && ids[j] == i) v = (dG[j] - gdg) / S * sg[j] * (1.f - sg[j]);
      dcrow[i] = v;
    }
    return;
  }

  // ---- noisy top-k softmax gate: dH_i = G_i (dG_i - sum_l G_l dG_l) on the kept
  float dHk[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) dHk[j] = gs[j] * (dG[j] - gdg);

  // load loss: P_i = Phi(u_i), u_i = (c_i - thr_i) / s_i; thr_i is H of the
  // (k+1)-th ranked expert jk1 when i is kept, of the k-th (jk) otherwise
  const bool loadg = a.noise && a.has_load;
  float thr_kept = -INFINITY, thr_out = -INFINITY;
  int jk1 = -1, jkk = 0;  // the (k+1)-th and the k-th ranked expert
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j == k - 1) jkk = ids[j];
  if (loadg) {
    const int4 q = a.kth[t];
    thr_kept = __int_as_float(q.x);
    jk1 = thr_kept == -INFINITY ? -1 : q.y;
    thr_out = __int_as_float(q.z);
  }
  auto kept_slot = [&](int i) {
    int js = -1;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k && ids[j] == i) js = j;
    return js;
  };
  // A_kept / A_out: sum of lam_load_i phi(u_i) / s_i over kept / not kept i
  float A_kept = 0.f, A_out = 0.f;
  if (loadg) {
    for (int i = lane; i < n; i += 32) {
      const bool kept = kept_slot(i) >= 0;
      const float thr = kept ? thr_kept : thr_out;
      const float sv = srow[i];
      if (thr == -INFINITY || sv == 0.f) continue;  // P constant there
      const float u = (crow[i] - thr) / sv;
      const float av = rc.lam_load[i] * (0.3989422804014327f * expf(-0.5f * u * u)) / sv;
      if (kept) A_kept += av; else A_out += av;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      A_kept += __shfl_xor_sync(0xffffffffu, A_kept, off);
      A_out += __shfl_xor_sync(0xffffffffu, A_out, off);
    }
  }
  const unsigned long long seed = a.seed_dev ? __ldg(a.seed_dev) : a.seed;
  const uint32_t key0 = (uint32_t)(seed & 0xffffffffu), key1 = (uint32_t)(seed >> 32);
  for (int m = lane; 4 * m < n; m += 32) {
    float eps[4] = {0.f, 0.f, 0.f, 0.f};
    if (a.noise) {
      const uint4 wd =
          philox4x32_10(make_uint4(rc.tok, (uint32_t)m, rc.gate_id, 0u), key0, key1);
      box_muller2(wd.x, wd.y, eps[0], eps[1]);
      box_muller2(wd.z, wd.w, eps[2], eps[3]);
    }
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const int i = 4 * m + j4;
      if (i >= n) break;
      const int js = kept_slot(i);
      float dH = 0.f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j == js) dH = dHk[j];
      float dc = 0.f, ds = 0.f;
      const float sv = a.noise ? srow[i] : 0.f;
      if (loadg) {
        if (i == jk1) dH -= A_kept;
        if (i == jkk) dH -= A_out;
        const float thr = js >= 0 ? thr_kept : thr_out;
        if (thr != -INFINITY && sv != 0.f) {
          const float u = (crow[i] - thr) / sv;
          const float av = rc.lam_load[i] * (0.3989422804014327f * expf(-0.5f * u * u)) / sv;
          dc += av;
          ds -= av * u;
        }
      }
      dc += dH;  // H = c + eps s
      dcrow[i] = dc;
      if (dzrow) {
        ds = fmaf(dH, eps[j4], ds);
        // s = Softplus(z): dz = ds Sigmoid(z), Sigmoid(z) = 1 - e^-s
        dzrow[i] = ds * -expm1f(-sv);
      }
    }
  }
}

// The noisy top-k gate's backward with the row in registers: lane l holds
// column quads l, l+32, ... (NQ of them, n <= 128 NQ, n a multiple of 4),
// loaded once with 16-byte loads, so both passes run from registers.  Same
// arithmetic, in the same order per element, as gate_bwd_kernel.
template <int KM, int NQ>
__global__ void __launch_bounds__(GW * 32) gate_bwd_reg_kernel(GateBwdArgs a) {
  const int t = blockIdx.x * GW + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int lane = threadIdx.x & 31;
  const int n = a.n, k = a.k;
  const RowCtx rc = row_ctx(a, t);
  const float4 *crow = reinterpret_cast<const float4 *>(a.c + (size_t)t * n);
  const float4 *srow = reinterpret_cast<const float4 *>(a.s + (size_t)t * n);
  float cv[NQ][4], sv[NQ][4];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int m = lane + 32 * q;
    float4 c4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = c4;
    if (4 * m < n) {
      c4 = __ldg(crow + m);
      if (a.noise) s4 = __ldg(srow + m);
    }
    cv[q][0] = c4.x; cv[q][1] = c4.y; cv[q][2] = c4.z; cv[q][3] = c4.w;
    sv[q][0] = s4.x; sv[q][1] = s4.y; sv[q][2] = s4.z; sv[q][3] = s4.w;
  }
  int ids[KM];
  float gs[KM], dG[KM];
  {
    int id = 0;
    float gv = 0.f, dv = 0.f;
    if (lane < k) {
      id = a.idx[(size_t)t * k + lane];
      gv = a.gate[(size_t)t * k + lane];
      // + the importance term (an id out of range, only after non-finite
      // logits, which the forward reports, reads nothing)
      dv = a.dgate[(size_t)t * k + lane] + (a.lam_imp && id >= 0 && id < n ? a.lam_imp[id] : 0.f);
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      ids[j] = __shfl_sync(0xffffffffu, id, j);
      gs[j] = __shfl_sync(0xffffffffu, gv, j);
      dG[j] = __shfl_sync(0xffffffffu, dv, j);
    }
  }
  float gdg = 0.f;
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j < k) gdg = fmaf(gs[j], dG[j], gdg);
  float dHk[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) dHk[j] = gs[j] * (dG[j] - gdg);
  int jkk = 0;
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j == k - 1) jkk = ids[j];
  const bool loadg = a.noise && a.has_load;
  float thr_kept = -INFINITY, thr_out = -INFINITY;
  int jk1 = -1;
  if (loadg) {
    const int4 q = a.kth[t];
    thr_kept = __int_as_float(q.x);
    jk1 = thr_kept == -INFINITY ? -1 : q.y;
    thr_out = __int_as_float(q.z);
  }
  auto kept_slot = [&](int i) {
    int js = -1;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k && ids[j] == i) js = j;
    return js;
  };
  // load term per element: av = lam_load_i phi(u_i) / s_i, u_i = (c_i - thr_i) / s_i
  float av[NQ][4], uv[NQ][4];
  float A_kept = 0.f, A_out = 0.f;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int i0 = 4 * (lane + 32 * q);
    float lam4[4] = {0.f, 0.f, 0.f, 0.f};
    if (loadg && i0 < n) {
      const float4 l4 = __ldg(reinterpret_cast<const float4 *>(rc.lam_load) + lane + 32 * q);
      lam4[0] = l4.x; lam4[1] = l4.y; lam4[2] = l4.z; lam4[3] = l4.w;
    }
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const int i = i0 + j4;
      av[q][j4] = 0.f;
      uv[q][j4] = 0.f;
      if (!loadg || i >= n) continue;
      const bool kept = kept_slot(i) >= 0;
      const float thr = kept ? thr_kept : thr_out;
      const float svv = sv[q][j4];
      if (thr == -INFINITY || svv == 0.f) continue;  // P constant there
      const float u = (cv[q][j4] - thr) / svv;
      const float v = lam4[j4] * (0.3989422804014327f * expf(-0.5f * u * u)) / svv;
      av[q][j4] = v;
      uv[q][j4] = u;
      if (kept) A_kept += v; else A_out += v;
    }
  }
  if (loadg) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      A_kept += __shfl_xor_sync(0xffffffffu, A_kept, off);
      A_out += __shfl_xor_sync(0xffffffffu, A_out, off);
    }
  }
  const unsigned long long seed = a.seed_dev ? __ldg(a.seed_dev) : a.seed;
  const uint32_t key0 = (uint32_t)(seed & 0xffffffffu), key1 = (uint32_t)(seed >> 32);
  float4 *dcrow = reinterpret_cast<float4 *>(a.dc + (size_t)t * n);
  float4 *dzrow = a.dz ? reinterpret_cast<float4 *>(a.dz + (size_t)t * n) : nullptr;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int m = lane + 32 * q;
    if (4 * m >= n) break;
    float eps[4] = {0.f, 0.f, 0.f, 0.f};
    if (a.noise) {
      const uint4 wd =
          philox4x32_10(make_uint4(rc.tok, (uint32_t)m, rc.gate_id, 0u), key0, key1);
      box_muller2(wd.x, wd.y, eps[0], eps[1]);
      box_muller2(wd.z, wd.w, eps[2], eps[3]);
    }
    float dc4[4], dz4[4];
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const int i = 4 * m + j4;
      const int js = kept_slot(i);
      float dH = 0.f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j == js) dH = dHk[j];
      float dc = 0.f, ds = 0.f;
      if (loadg) {
        if (i == jk1) dH -= A_kept;
        if (i == jkk) dH -= A_out;
        dc += av[q][j4];
        ds -= av[q][j4] * uv[q][j4];
      }
      dc += dH;  // H = c + eps s
      dc4[j4] = dc;
      ds = fmaf(dH, eps[j4], ds);
      // s = Softplus(z): dz = ds Sigmoid(z), Sigmoid(z) = 1 - e^-s
      dz4[j4] = ds * -expm1f(-sv[q][j4]);
    }
    dcrow[m] = make_float4(dc4[0], dc4[1], dc4[2], dc4[3]);
    if (dzrow) dzrow[m] = make_float4(dz4[0], dz4[1], dz4[2], dz4[3]);
  }
}

// ---------------------------------------------------------------- gate_stats_bwd
// The router z-loss w_z mean_t |c_t|^2 and the gate entropy term
// -w_entropy mean_t H(softmax(c_t)) ([MoE-intro] 第三部分): per token (warp),
// an online pass for m = max c, S = sum e^(c-m), Q = sum e^(c-m) (c-m)
// (H = log S - Q/S), then dc_i += (w_z 2 c_i + w_entropy p_i (log p_i + H)) / T,
// since dH/dc_i = -p_i (log p_i + H).
__global__ void __launch_bounds__(GW * 32) gate_stats_bwd_kernel(const float *__restrict__ c,
                                                                  int T, int n, float w_z,
                                                                  float w_e, float *dc) {
  const int t = blockIdx.x * GW + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  const float *crow = c + (size_t)t * n;
  float m = -INFINITY, S = 0.f, Q = 0.f;
  for (int i = lane; i < n; i += 32) {
    const float v = crow[i];
    if (v > m) {  // rescale to the new maximum
      const float r = S > 0.f ? expf(m - v) : 0.f;
      Q = S > 0.f ? r * (Q + S * (m - v)) : 0.f;
      S *= r;
      m = v;
    }
    const float e = expf(v - m);
    S += e;
    Q = fmaf(e, v - m, Q);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, off);
    const float os = __shfl_xor_sync(0xffffffffu, S, off);
    const float oq = __shfl_xor_sync(0xffffffffu, Q, off);
    const float m2 = fmaxf(m, om);
    const float r1 = S > 0.f ? expf(m - m2) : 0.f, r2 = os > 0.f ? expf(om - m2) : 0.f;
    Q = (S > 0.f ? r1 * (Q + S * (m - m2)) : 0.f) + (os > 0.f ? r2 * (oq + os * (om - m2)) : 0.f);
    S = S * r1 + os * r2;
    m = m2;
  }
  const float logS = logf(S), H = logS - Q / S, invT = 1.f / (float)T;
  float *drow = dc + (size_t)t * n;
  for (int i = lane; i < n; i += 32) {
    const float v = crow[i];
    const float lp = v - m - logS;
    drow[i] += (w_z * 2.f * v + w_e * expf(lp) * (lp + H)) * invT;
  }
}

// ---------------------------------------------------------------- colsum
// part[blockIdx.y][j] = sum of rows [blockIdx.y * rows_per, ...) of column j
__global__ void __launch_bounds__(256) colsum_kernel(const float *__restrict__ X, int R, int N,
                                                     int rows_per, float *__restrict__ part) {
  const int j = blockIdx.x * 256 + threadIdx.x;
  if (j >= N) return;
  const int r0 = blockIdx.y * rows_per, r1 = min(r0 + rows_per, R);
  float s = 0.f;
#pragma unroll 4
  for (int r = r0; r < r1; ++r) s += __ldg(X + (size_t)r * N + j);
  part[(size_t)blockIdx.y * N + j] = s;
}

}  // namespace

int launch_bwd_coef(const float *importance, const float *load, const int *counts, int n, int T,
                    float w_imp, float w_load, float alpha, int router, int noise, float *lam_imp,
                    float *lam_load, float *sw_coef, cudaStream_t st) {
  return launch("bwd_coef", bwd_coef_kernel, dim3(1), dim3(CT), 0, st, importance, load, counts,
                n, T, w_imp, w_load, alpha, router, noise, lam_imp, lam_load, sw_coef);
}

int launch_combine_bwd(const float *dy, const float *gate, const int *row_of, const void *y_perm,
                       int bf16, int T, int k, int d, void *dy_perm, float *dgate, void *dy_shared,
                       cudaStream_t st) {
  if (k > kMaxK) return MOE_EINVAL;
  const dim3 grid((unsigned)ceil_div(T, NT / 32));
  auto go = [&](auto kern) {
    return launch("combine_bwd", kern, grid, dim3(NT), 0, st, dy, gate, row_of, y_perm, T, k, d,
                  dy_perm, dgate, dy_shared);
  };
  if (bf16) {
    if (k <= 1) return go(combine_bwd_kernel<1, true>);
    if (k <= 2) return go(combine_bwd_kernel<2, true>);
    if (k <= 4) return go(combine_bwd_kernel<4, true>);
    return go(combine_bwd_kernel<8, true>);
  }
  if (k <= 1) return go(combine_bwd_kernel<1, false>);
  if (k <= 2) return go(combine_bwd_kernel<2, false>);
  if (k <= 4) return go(combine_bwd_kernel<4, false>);
  return go(combine_bwd_kernel<8, false>);
}

int launch_expert_bwd_f32(const float *x_perm, const float *dy_perm, const int *offsets, int n,
                          int d, int f, const float *W1, const float *b1, const float *W2,
                          float *dx_perm, float *dW1, float *db1, float *dW2, float *db2,
                          const char *name, cudaStream_t st) {
  const size_t smem = sizeof(float) * (size_t)(2 * d + 2 * f);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(expert_bwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_EINVAL;
  return launch(name ? name : "expert_bwd_fp32", expert_bwd_f32_kernel, dim3((unsigned)n),
                dim3(256), smem, st, x_perm, dy_perm, offsets, d, f, W1, b1, W2, dx_perm, dW1, db1,
                dW2, db2);
}

int launch_dx_gather(const void *dx_perm, int bf16, const int *row_of, const float *dy,
                     int passthrough, int T, int k, int d, const void *dx_shared, float *dx,
                     cudaStream_t st) {
  if (k > kMaxK) return MOE_EINVAL;
  const dim3 grid((unsigned)ceil_div(T, NT / 32));
  auto go = [&](auto kern) {
    return launch("dx_gather", kern, grid, dim3(NT), 0, st, dx_perm, row_of, dy, passthrough, T,
                  k, d, dx_shared, dx);
  };
  if (bf16) {
    if (k <= 1) return go(dx_gather_kernel<1, true>);
    if (k <= 2) return go(dx_gather_kernel<2, true>);
    if (k <= 4) return go(dx_gather_kernel<4, true>);
    return go(dx_gather_kernel<8, true>);
  }
  if (k <= 1) return go(dx_gather_kernel<1, false>);
  if (k <= 2) return go(dx_gather_kernel<2, false>);
  if (k <= 4) return go(dx_gather_kernel<4, false>);
  return go(dx_gather_kernel<8, false>);
}

int launch_bias_grad(const void *dy_perm, const void *dhid, const int *offsets, int n, int d,
                     int f, float *db2, float *db1, const char *name, cudaStream_t st) {
  const dim3 grid((unsigned)(ceil_div(d, 256) + ceil_div(f, 256)), (unsigned)n);
  return launch(name ? name : "bias_grad", bias_grad_kernel, grid, dim3(256), 0, st,
                static_cast<const __nv_bfloat16 *>(dy_perm),
                static_cast<const __nv_bfloat16 *>(dhid), offsets, d, f, db2, db1);
}

int launch_gate_bwd(const GateBwdArgs &a, cudaStream_t st) {
  if (a.k > kMaxK) return MOE_EINVAL;
  const dim3 grid((unsigned)ceil_div(a.T, GW));
  auto go = [&](auto kern) { return launch("gate_bwd", kern, grid, dim3(GW * 32), 0, st, a); };
  if (a.router == MOE_ROUTER_NOISY_TOPK && (a.n & 3) == 0 && a.n <= 4 * 32 * 8) {
    // the row in registers: quads per lane 1, 2, 4 or 8
    const int nq = (a.n + 127) / 128;
#define MOE_GBWD_REG(KMV)                                                      \
    if (nq <= 1) return go(gate_bwd_reg_kernel<KMV, 1>);                       \
    if (nq <= 2) return go(gate_bwd_reg_kernel<KMV, 2>);                       \
    if (nq <= 4) return go(gate_bwd_reg_kernel<KMV, 4>);                       \
    return go(gate_bwd_reg_kernel<KMV, 8>);
    if (a.k <= 1) { MOE_GBWD_REG(1) }
    if (a.k <= 2) { MOE_GBWD_REG(2) }
    if (a.k <= 4) { MOE_GBWD_REG(4) }
    MOE_GBWD_REG(8)
#undef MOE_GBWD_REG
  }
  if (a.k <= 1) return go(gate_bwd_kernel<1>);
  if (a.k <= 2) return go(gate_bwd_kernel<2>);
  if (a.k <= 4) return go(gate_bwd_kernel<4>);
  return go(gate_bwd_kernel<8>);
}

// row blocks of at least 16 rows, about two blocks per SM over all column blocks
int launch_gate_stats_bwd(const float *c, int T, int n, float w_z, float w_entropy, float *dc,
                          cudaStream_t st) {
  return launch("gate_stats_bwd", gate_stats_bwd_kernel, dim3((unsigned)ceil_div(T, GW)),
                dim3(GW * 32), 0, st, c, T, n, w_z, w_entropy, dc);
}

int colsum_parts(int R, int N) {
  if (R <= 0) return 0;
  const int cb = (int)ceil_div(N, 256);
  const int want = (int)ceil_div(2 * num_sms(), cb);
  const int most = (int)ceil_div(R, 16);
  return want < most ? (want > 0 ? want : 1) : most;
}

int launch_colsum(const float *X, int R, int N, float *part, float *out, cudaStream_t st) {
  const int parts = colsum_parts(R, N);
  if (parts == 0) {
    return cudaMemsetAsync(out, 0, 4 * (size_t)N, st) == cudaSuccess ? MOE_OK : MOE_ECUDA;
  }
  const int rows_per = (int)ceil_div(R, parts);
  MOE_TRY(launch("colsum", colsum_kernel, dim3((unsigned)ceil_div(N, 256), (unsigned)parts),
                 dim3(256), 0, st, X, R, N, rows_per, part));
  return launch_route_reduce(part, nullptr, 1, parts, N, out, st);
}

}  // namespace moe
