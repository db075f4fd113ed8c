// combine.cu -- y = sum_i G(x)_i E_i(x) ([SGMoE-note] "Sparsely-Gated MoE 层架构")
// over each token's kept slots, in slot order, fp32 accumulation.  A dropped
// slot adds nothing; a token with no kept slot passes through the residual
// ([MoE-deep] §3.2) when pass-through is on (y = x), else gets 0.  With a
// shared expert ([MoE-deep] §5.2) its row E_shared(x) is the first term of
// every token's sum (and is added to the pass-through x).
// One warp per token, 8 features per lane per step: the 16-byte loads of all
// the token's expert rows are issued before the sums, two 16-byte stores of y.
#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

// KM: slots per token rounded up to 1, 2, 4 or 8 (register arrays sized by it)
template <bool BF16, int KM>
__global__ void __launch_bounds__(NT) combine_kernel(const void *__restrict__ yp,
                                                      const float *__restrict__ gate,
                                                      const int *__restrict__ row_of,
                                                      const float *__restrict__ x, int passthrough,
                                                      int T, int k, int d, float *__restrict__ y,
                                                      const void *__restrict__ ys) {
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int rows[KM];
  float g[KM];
  bool any = false;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    rows[j] = j < k ? __ldg(row_of + (size_t)t * k + j) : -1;
    g[j] = j < k ? __ldg(gate + (size_t)t * k + j) : 0.f;
    any |= rows[j] >= 0;
  }
  float4 *yr = reinterpret_cast<float4 *>(y + (size_t)t * d);
  const int nchunk = d >> 3;
  // the shared expert's 8 features of chunk c of this token (0 without one)
  auto shared8 = [&](int c, float (&s)[8]) {
    if (!ys) {
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] = 0.f;
    } else if (BF16) {
      const uint4 pk = __ldg(reinterpret_cast<const uint4 *>(
                                 static_cast<const __nv_bfloat16 *>(ys) + (size_t)t * d) + c);
      const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[u]));
        s[2 * u] = f2.x;
        s[2 * u + 1] = f2.y;
      }
    } else {
      const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(ys) + (size_t)t * d);
      const float4 u = __ldg(src + 2 * c), v = __ldg(src + 2 * c + 1);
      s[0] = u.x; s[1] = u.y; s[2] = u.z; s[3] = u.w;
      s[4] = v.x; s[5] = v.y; s[6] = v.z; s[7] = v.w;
    }
  };
  if (!any) {
    const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)t * d);
    for (int c = lane; c < nchunk; c += 32) {
      float4 u = make_float4(0.f, 0.f, 0.f, 0.f), v = u;
      if (passthrough) {
        u = __ldg(xr + 2 * c);
        v = __ldg(xr + 2 * c + 1);
      }
      if (ys) {
        float s[8];
        shared8(c, s);
        u.x += s[0]; u.y += s[1]; u.z += s[2]; u.w += s[3];
        v.x += s[4]; v.y += s[5]; v.z += s[6]; v.w += s[7];
      }
      yr[2 * c] = u;
      yr[2 * c + 1] = v;
    }
    return;
  }
  constexpr int UNR = KM <= 4 ? 2 : 1;  // two chunks in flight while registers allow
#pragma unroll UNR
  for (int c = lane; c < nchunk; c += 32) {
    // every kept slot's 8 features first (independent loads), then the sum
    float f[KM][8];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (rows[j] < 0) continue;
      if (BF16) {
        const uint4 pk = __ldg(reinterpret_cast<const uint4 *>(
                                   static_cast<const __nv_bfloat16 *>(yp) + (size_t)rows[j] * d) +
                               c);
        const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[u]));
          f[j][2 * u] = f2.x;
          f[j][2 * u + 1] = f2.y;
        }
      } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(yp) +
                                                             (size_t)rows[j] * d);
        const float4 u = __ldg(src + 2 * c), v = __ldg(src + 2 * c + 1);
        f[j][0] = u.x; f[j][1] = u.y; f[j][2] = u.z; f[j][3] = u.w;
        f[j][4] = v.x; f[j][5] = v.y; f[j][6] = v.z; f[j][7] = v.w;
      }
    }
    float acc[8];
    shared8(c, acc);
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (rows[j] < 0) continue;
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = fmaf(g[j], f[j][u], acc[u]);
    }
    yr[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    yr[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

int launch_combine(const void *y_perm, int bf16, const float *gate, const int *row_of,
                   const float *x, int passthrough, int T, int k, int d, float *y,
                   const void *y_shared, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(T, NT / 32));
  auto go = [&](auto kern) {
    return launch("combine", kern, grid, dim3(NT), 0, st, y_perm, gate, row_of, x, passthrough, T,
                  k, d, y, y_shared);
  };
  if (k > kMaxK) return MOE_EINVAL;
  if (bf16) {
    if (k <= 1) return go(combine_kernel<true, 1>);
    if (k <= 2) return go(combine_kernel<true, 2>);
    if (k <= 4) return go(combine_kernel<true, 4>);
    return go(combine_kernel<true, 8>);
  }
  if (k <= 1) return go(combine_kernel<false, 1>);
  if (k <= 2) return go(combine_kernel<false, 2>);
  if (k <= 4) return go(combine_kernel<false, 4>);
  return go(combine_kernel<false, 8>);
}

}  // namespace moe
