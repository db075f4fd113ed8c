// stats.cu -- the balancing statistics.
//   Importance(X)_i = sum_x G(x)_i                 ([SGMoE-xyz] "負載平衡損失")
//   L_importance = w_importance * CV(Importance)^2, L_load = w_load * CV(Load)^2
//   Switch: N * sum_i f_i P_i, f_i = count_i / T, P_i = mean router prob
//           ([MoE-deep] §3.2), and alpha times it
//   drop rate = slots beyond capacity / (T k)
// Importance is a segmented sum over the gates already sorted by expert by
// the dispatch (one warp per expert, fixed order); the scalar losses are one
// block in fp64 (CV^2 of a near-uniform vector cancels badly in fp32).
#include "internal.h"

namespace moe {
namespace {

__global__ void importance_kernel(const float *gate_sorted, const int *ucoff, int n,
                                  float *importance) {
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= n) return;
  const int lane = threadIdx.x & 31;
  const int p0 = ucoff[e], p1 = ucoff[e + 1];
  float s = 0.f;
  for (int p = p0 + lane; p < p1; p += 32) s += gate_sorted[p];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) importance[e] = s;
}

constexpr int LNT = 1024;

// fixed-order block reduction of one double per thread
__device__ double block_sum(double v, double *sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) sh[w] = v;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < LNT / 32; ++i) r += sh[i];
  __syncthreads();
  if (threadIdx.x == 0) sh[0] = r;
  __syncthreads();
  r = sh[0];
  __syncthreads();
  return r;
}

__device__ double cv2(const float *v, int n, double *sh) {
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += LNT) s += (double)v[i];
  const double mean = block_sum(s, sh) / (double)n;
  if (mean == 0.0) return 0.0;
  double q = 0.0;
  for (int i = threadIdx.x; i < n; i += LNT) {
    const double dv = (double)v[i] - mean;
    q += dv * dv;
  }
  const double var = block_sum(q, sh) / (double)n;
  return var / (mean * mean);
}

__global__ void __launch_bounds__(LNT) losses_kernel(const float *importance, const float *load,
                                                     const int *counts, const float *prob_sum,
                                                     int n, int T, int k, long long C, int router,
                                                     float w_imp, float w_load, float alpha,
                                                     const float *rstats, const float *dropped_in,
                                                     float *losses) {
  __shared__ double sh[LNT / 32];
  const double cv_imp = cv2(importance, n, sh);
  const double cv_load = cv2(load, n, sh);
  double aux_part = 0.0, drop_part = 0.0;
  for (int i = threadIdx.x; i < n; i += LNT) {
    const long long c = counts[i];
    if (c > C) drop_part += (double)(c - C);
    if (router == MOE_ROUTER_SWITCH && prob_sum && T > 0)
      aux_part += ((double)c / (double)T) * ((double)prob_sum[i] / (double)T);
  }
  const double aux = block_sum(aux_part, sh) * (double)n;
  // with dropped_in the dropped slots were counted elsewhere (the shards of
  // an expert-parallel batch each cut at their own capacity)
  const double dropped = dropped_in ? (double)*dropped_in : block_sum(drop_part, sh);
  if (threadIdx.x == 0) {
    const double S = (double)T * (double)k;
    losses[0] = (float)((double)w_imp * cv_imp);
    losses[1] = (float)((double)w_load * cv_load);
    losses[2] = (float)aux;
    losses[3] = (float)((double)alpha * aux);
    losses[4] = (float)(S > 0 ? dropped / S : 0.0);
    losses[5] = (float)cv_imp;
    losses[6] = (float)cv_load;
    losses[7] = (float)dropped;
    // router statistics: means over tokens of |c|^2 and of the softmax entropy
    losses[8] = rstats && T > 0 ? (float)((double)rstats[0] / T) : 0.f;
    losses[9] = rstats && T > 0 ? (float)((double)rstats[1] / T) : 0.f;
  }
}

// Selection-bias update of the sigmoid router ([MoE-deep] §6.3): overloaded
// experts (more than T*k/n slots, compared exactly as counts*n > T*k) lose
// gamma, underloaded ones gain it, fp32.
__global__ void sel_bias_update_kernel(const int *counts, int n, long long total, float gamma,
                                       float *bias) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const long long scaled = (long long)counts[i] * n;
  if (scaled > total) bias[i] = bias[i] - gamma;
  else if (scaled < total) bias[i] = bias[i] + gamma;
}

// The next noise key: one add in stream order, so a captured graph that
// starts with it draws new noise at every replay.
__global__ void noise_step_kernel(unsigned long long *seed) { *seed += 1ull; }

}  // namespace

int launch_noise_step(unsigned long long *seed, cudaStream_t st) {
  return launch("noise_step", noise_step_kernel, dim3(1), dim3(1), 0, st, seed);
}

int launch_sel_bias_update(const int *counts, int n, int T, int k, float gamma, float *bias,
                           cudaStream_t st) {
  return launch("sel_bias_update", sel_bias_update_kernel, dim3((unsigned)ceil_div(n, 256)),
                dim3(256), 0, st, counts, n, (long long)T * k, gamma, bias);
}

int launch_importance(const float *gate_sorted, const int *ucoff, int n, float *importance,
                      cudaStream_t st) {
  return launch("importance", importance_kernel, dim3((unsigned)ceil_div(n, 8)), dim3(256), 0, st,
                gate_sorted, ucoff, n, importance);
}

int launch_losses(const float *importance, const float *load, const int *counts,
                  const float *prob_sum, int n, int T, int k, int64_t C, int router, float w_imp,
                  float w_load, float alpha, const float *rstats, float *losses, cudaStream_t st,
                  const float *dropped) {
  return launch("balance_losses", losses_kernel, dim3(1), dim3(LNT), 0, st, importance, load,
                counts, prob_sum, n, T, k, (long long)C, router, w_imp, w_load, alpha, rstats,
                dropped, losses);
}

}  // namespace moe
