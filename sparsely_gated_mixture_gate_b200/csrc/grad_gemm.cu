// grad_gemm.cu -- fp32 GEMMs of the gate's backward pass on the CUDA cores.
//
// The gate stays in fp32 ([SGMoE-note] 缺点与局限性: the layer diverges when
// trained in bf16), so its gradients are fp32 contractions:
//   dW_g = x^T dc, dW_noise = x^T dz        (M = d, N = n, K = T)
//   dx  += dc W_g^T + dz W_noise^T          (M = T, N = d, K = n)
// One kernel for both shapes: C[M][N] = sum_k A(m,k) B(k,n), A and B read
// row- or column-major, 128x128 tiles of 256 threads (8x8 outputs each),
// 8-deep K slices staged through double-buffered shared memory.  When M x N
// is small next to the machine (the weight gradients: K = T is the long
// side) the K range is split across CTAs into a scratch buffer, and a second
// kernel adds the splits in order, so the result does not depend on timing.
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 128, BK = 8, NT = 256;

// element (r, c) of an R x Cc view of a matrix stored row-major with leading
// dimension ld, or transposed (stored Cc x R)
template <bool TR>
__device__ __forceinline__ float ld_elem(const float *__restrict__ p, int ld, int r, int c) {
  return TR ? __ldg(p + (size_t)c * ld + r) : __ldg(p + (size_t)r * ld + c);
}

template <bool AT, bool BT>
__global__ void __launch_bounds__(NT) sgemm_kernel(SgemmArgs a) {
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BN + 4];
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int splits = a.part ? a.splits : 1;
  const int kc = (a.K + splits - 1) / splits;
  const int kbeg = blockIdx.z * kc, kend = min(a.K, kbeg + kc);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

  // loader mapping: 256 threads x 4 elements = a 128 x 8 slice.  Stored
  // [M][K] (A not transposed): thread -> (row tid>>1, 4 columns (tid&1)*4);
  // stored [K][M]: thread -> (k-row tid>>5, 4 columns (tid&31)*4).
  float ra[4], rb[4];
  auto load_a = [&](int k0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int m, kk;
      if (!AT) { m = m0 + (tid >> 1); kk = k0 + (tid & 1) * 4 + u; }
      else { m = m0 + (tid & 31) * 4 + u; kk = k0 + (tid >> 5); }
      ra[u] = (m < a.M && kk < kend) ? (AT ? ld_elem<true>(a.A, a.lda, m, kk)
                                          : ld_elem<false>(a.A, a.lda, m, kk))
                                     : 0.f;
    }
  };
  auto load_b = [&](int k0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int nn, kk;
      if (BT) { nn = n0 + (tid >> 1); kk = k0 + (tid & 1) * 4 + u; }
      else { nn = n0 + (tid & 31) * 4 + u; kk = k0 + (tid >> 5); }
      // B(k, n): stored [K][N] (row k), or [N][K] with bt
      rb[u] = (nn < a.N && kk < kend) ? (BT ? __ldg(a.B + (size_t)nn * a.ldb + kk)
                                            : __ldg(a.B + (size_t)kk * a.ldb + nn))
                                      : 0.f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!AT) As[buf][(tid & 1) * 4 + u][tid >> 1] = ra[u];
      else As[buf][tid >> 5][(tid & 31) * 4 + u] = ra[u];
      if (BT) Bs[buf][(tid & 1) * 4 + u][tid >> 1] = rb[u];
      else Bs[buf][tid >> 5][(tid & 31) * 4 + u] = rb[u];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  int buf = 0;
  if (kbeg < kend) {
    load_a(kbeg);
    load_b(kbeg);
    store(0);
    __syncthreads();
    for (int k0 = kbeg; k0 < kend; k0 += BK) {
      const bool more = k0 + BK < kend;
      if (more) {  // next slice into registers while this one is used
        load_a(k0 + BK);
        load_b(k0 + BK);
      }
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 8]);
        const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 8 + 4]);
        const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 8]);
        const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 8 + 4]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      if (more) {
        store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

  // rows ty*8.., columns tx*8..
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
    if (m >= a.M) break;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int nn = n0 + tx * 8 + j;
      if (nn >= a.N) break;
      if (a.part) {
        a.part[((size_t)blockIdx.z * a.M + m) * a.N + nn] = acc[i][j];
      } else {
        float *c = a.C + (size_t)m * a.ldc + nn;
        *c = a.accumulate ? *c + acc[i][j] : acc[i][j];
      }
    }
  }
}

// C = sum over the splits in order (+ C)
__global__ void __launch_bounds__(256) split_sum_kernel(const float *__restrict__ part, int splits,
                                                        int M, int N, float *C, int ldc,
                                                        int accumulate) {
  const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= (size_t)M * N) return;
  float s = 0.f;
  for (int z = 0; z < splits; ++z) s += part[(size_t)z * M * N + i];
  const int m = (int)(i / N), nn = (int)(i % N);
  float *c = C + (size_t)m * ldc + nn;
  *c = accumulate ? *c + s : s;
}

}  // namespace

int sgemm_splits(int M, int N, int K) {
  const int tiles = (int)(ceil_div(M, BM) * ceil_div(N, BN));
  const int want = 2 * num_sms();
  if (tiles >= want / 2 || K < 8 * BK) return 1;
  int s = want / tiles;
  const int smax = (int)ceil_div(K, 4 * BK);  // at least 4 slices per split
  if (s > smax) s = smax;
  return s < 1 ? 1 : s;
}

int launch_sgemm(const SgemmArgs &a, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0) return MOE_OK;
  SgemmArgs b = a;
  if (b.splits <= 1) b.part = nullptr;
  const int splits = b.part ? b.splits : 1;
  const dim3 grid((unsigned)ceil_div(a.N, BN), (unsigned)ceil_div(a.M, BM), (unsigned)splits);
  const char *name = a.name ? a.name : "gate_grad_gemm";
  int rc;
  if (!a.at && !a.bt) rc = launch(name, sgemm_kernel<false, false>, grid, dim3(NT), 0, st, b);
  else if (a.at && !a.bt) rc = launch(name, sgemm_kernel<true, false>, grid, dim3(NT), 0, st, b);
  else if (!a.at && a.bt) rc = launch(name, sgemm_kernel<false, true>, grid, dim3(NT), 0, st, b);
  else rc = launch(name, sgemm_kernel<true, true>, grid, dim3(NT), 0, st, b);
  if (rc != MOE_OK || !b.part) return rc;
  const size_t total = (size_t)a.M * a.N;
  return launch("gate_grad_split_sum", split_sum_kernel, dim3((unsigned)ceil_div((int64_t)total, 256)),
                dim3(256), 0, st, (const float *)b.part, splits, a.M, a.N, a.C, a.ldc,
                a.accumulate);
}

}  // namespace moe
