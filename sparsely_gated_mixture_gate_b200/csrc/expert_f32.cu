// expert_f32.cu -- fp32 experts (the tiny fp32 workload): the same ReLU FFN
// ([SGMoE-note] "Sparsely-Gated MoE 层架构") on the FP32 pipes.
//   y = ReLU(x W1_e^T + b1_e) W2_e^T + b2_e   for every kept row of expert e
// One block per row; the row and its hidden layer sit in shared memory; one
// warp per output feature, lanes striding over the contiguous weight row
// (coalesced), fixed-order shuffle reduction.
#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256, NWARP = NT / 32;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__global__ void __launch_bounds__(NT) expert_f32_kernel(const float *xp, const int *offsets, int n,
                                                         int d, int f, const float *W1,
                                                         const float *b1, const float *W2,
                                                         const float *b2, float *yp) {
  extern __shared__ float sh[];
  float *xs = sh;       // [d]
  float *hs = sh + d;   // [f]
  const int row = blockIdx.x;
  if (row >= offsets[n]) return;
  int lo = 0, hi = n - 1;  // expert: largest e with offsets[e] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  for (int q = threadIdx.x; q < d; q += NT) xs[q] = xp[(size_t)row * d + q];
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float *W1e = W1 + (size_t)e * f * d;
  for (int j = w; j < f; j += NWARP) {
    const float *wr = W1e + (size_t)j * d;
    float acc = 0.f;
    for (int q = lane; q < d; q += 32) acc = fmaf(xs[q], wr[q], acc);
    acc = warp_sum(acc);
    if (lane == 0) hs[j] = fmaxf(acc + (b1 ? b1[(size_t)e * f + j] : 0.f), 0.f);
  }
  __syncthreads();
  const float *W2e = W2 + (size_t)e * d * f;
  for (int q = w; q < d; q += NWARP) {
    const float *wr = W2e + (size_t)q * f;
    float acc = 0.f;
    for (int j = lane; j < f; j += 32) acc = fmaf(hs[j], wr[j], acc);
    acc = warp_sum(acc);
    if (lane == 0) yp[(size_t)row * d + q] = acc + (b2 ? b2[(size_t)e * d + q] : 0.f);
  }
}

}  // namespace

int launch_expert_f32(const ExpertArgs &a, cudaStream_t st) {
  if (a.S == 0) return MOE_OK;
  const size_t smem = sizeof(float) * (size_t)(a.d + a.f);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(expert_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_EINVAL;
  }
  return launch(a.name ? a.name : "expert_ffn_fp32", expert_f32_kernel, dim3(a.S), dim3(NT), smem, st,
                static_cast<const float *>(a.x_perm), a.offsets, a.n, a.d, a.f,
                static_cast<const float *>(a.W1), a.b1, static_cast<const float *>(a.W2), a.b2,
                static_cast<float *>(a.y_perm));
}

}  // namespace moe
