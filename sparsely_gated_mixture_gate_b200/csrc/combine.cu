// combine.cu -- y = sum_i G(x)_i E_i(x) ([SGMoE-note] "Sparsely-Gated MoE 层架构")
// over each token's kept slots, in slot order, fp32 accumulation.  A dropped
// slot adds nothing; a token with no kept slot passes through the residual
// ([MoE-deep] §3.2) when pass-through is on (y = x), else gets 0.
// One warp per token, 8 features per lane per step: 16-byte loads of the
// expert rows, two 16-byte stores of y.
#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

template <bool BF16>
__global__ void __launch_bounds__(NT) combine_kernel(const void *yp, const float *gate,
                                                      const int *row_of, const float *x,
                                                      int passthrough, int T, int k, int d,
                                                      float *y) {
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int rows[kMaxK];
  float g[kMaxK];
  bool any = false;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    rows[j] = j < k ? row_of[(size_t)t * k + j] : -1;
    g[j] = j < k ? gate[(size_t)t * k + j] : 0.f;
    any |= rows[j] >= 0;
  }
  float4 *yr = reinterpret_cast<float4 *>(y + (size_t)t * d);
  const int nchunk = d >> 3;
  for (int c = lane; c < nchunk; c += 32) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (!any && passthrough) {
      const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)t * d);
      const float4 u = __ldg(xr + 2 * c), v = __ldg(xr + 2 * c + 1);
      acc[0] = u.x; acc[1] = u.y; acc[2] = u.z; acc[3] = u.w;
      acc[4] = v.x; acc[5] = v.y; acc[6] = v.z; acc[7] = v.w;
    } else {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (rows[j] < 0) continue;
        if (BF16) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4 *>(
                                     static_cast<const __nv_bfloat16 *>(yp) + (size_t)rows[j] * d) +
                                 c);
          const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[u]));
            acc[2 * u] = fmaf(g[j], f2.x, acc[2 * u]);
            acc[2 * u + 1] = fmaf(g[j], f2.y, acc[2 * u + 1]);
          }
        } else {
          const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(yp) +
                                                               (size_t)rows[j] * d);
          const float4 u = __ldg(src + 2 * c), v = __ldg(src + 2 * c + 1);
          acc[0] = fmaf(g[j], u.x, acc[0]); acc[1] = fmaf(g[j], u.y, acc[1]);
          acc[2] = fmaf(g[j], u.z, acc[2]); acc[3] = fmaf(g[j], u.w, acc[3]);
          acc[4] = fmaf(g[j], v.x, acc[4]); acc[5] = fmaf(g[j], v.y, acc[5]);
          acc[6] = fmaf(g[j], v.z, acc[6]); acc[7] = fmaf(g[j], v.w, acc[7]);
        }
      }
    }
    yr[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    yr[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

int launch_combine(const void *y_perm, int bf16, const float *gate, const int *row_of,
                   const float *x, int passthrough, int T, int k, int d, float *y,
                   cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(T, NT / 32));
  if (bf16)
    return launch("combine", combine_kernel<true>, grid, dim3(NT), 0, st, y_perm, gate, row_of, x,
                  passthrough, T, k, d, y);
  return launch("combine", combine_kernel<false>, grid, dim3(NT), 0, st, y_perm, gate, row_of, x,
                passthrough, T, k, d, y);
}

}  // namespace moe
