// grad_gemm.cu -- fp32 GEMMs of the gate's backward pass on the CUDA cores.
//
// The gate stays in fp32 ([SGMoE-note] 缺点与局限性: the layer diverges when
// trained in bf16), so its gradients are fp32 contractions:
//   dW_g = x^T dc, dW_noise = x^T dz        (M = d, N = n, K = T; one launch,
//                                            two problems sharing A)
//   dx  += dc W_g^T + dz W_noise^T          (M = T, N = d, K = n; one launch,
//                                            the two products summed)
// One kernel for all of them: C[M][N] = sum over pairs p of sum_k A_p(m,k)
// B_p(k,n), A read row- or column-major, B likewise.  128 x 128 tiles, 16-deep
// K slices, 256 threads with 8 x 8 outputs each held as four 4 x 4 quadrants
// (rows ty*4 and 64+ty*4, columns tx*4 and 64+tx*4) so that the shared-memory
// reads of a warp are broadcasts or conflict free; 16-byte global loads where
// the layout allows, double-buffered shared memory.  When M x N is small next
// to the machine (the weight gradients: K = T is the long side) the K range
// is split across CTAs into a scratch buffer and a second kernel adds the
// splits in order, so the result does not depend on timing.
// A grouped mode serves the hierarchical layer's secondary gates: one launch
// over the groups' row segments, along K (the weight gradients, A's rows
// gathered by token) or along M (the input gradient, one weight pair per group).
#include "fma2.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 128, BK = 16, NT = 256;
static_assert(BM == kGateBM, "grouped M tiles come from the gate's 128-row tile prefix");

// GR: the grouped mode (compiled separately so that the plain instances keep
// their registers)
template <bool AT, bool BT, bool GR>
__global__ void __launch_bounds__(NT, 2) sgemm_kernel(SgemmArgs a) {
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BN + 4];
  int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int splits = a.part ? a.splits : 1;
  int prob = a.nprob > 1 ? (int)blockIdx.z / splits : 0;
  const int split = (int)blockIdx.z % splits;
  // split length a multiple of the slice, so every 16-byte load stays aligned
  const int kc = (a.K + splits - 1) / splits + BK - 1 & ~(BK - 1);
  int kbeg = split * kc, kend = min(a.K, kbeg + kc);
  int Mx = a.M;                   // rows of this problem
  const int *arow = nullptr;      // A's rows (stored [K][M]) gathered through it
  int64_t offA = 0, offB = 0, offC = 0;
  if (GR) {
    if (a.seg_k) {  // blockIdx.z = group * nprob + problem
      const int g = (int)blockIdx.z / a.nprob;
      prob = (int)blockIdx.z % a.nprob;
      const int r0 = a.seg_off[g];
      kbeg = 0;
      kend = a.seg_off[g + 1] - r0;
      arow = a.a_row + r0;
      offB = (int64_t)r0 * a.ldb;
      offC = (int64_t)g * a.sC;
    } else {  // blockIdx.y = the M tile over all groups
      const int t = (int)blockIdx.y;
      if (t >= a.seg_mblk[a.G]) return;
      int lo = 0, hi = a.G - 1;  // largest g with seg_mblk[g] <= t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.seg_mblk[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int r0 = a.seg_off[lo];
      m0 = (t - a.seg_mblk[lo]) * BM;
      Mx = a.seg_off[lo + 1] - r0;
      offA = (int64_t)r0 * a.lda;
      offB = (int64_t)lo * a.sB;
      offC = (int64_t)r0 * a.ldc;
    }
  }
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // 16-byte loads need 4 consecutive in-range elements along the contiguous
  // dimension and a leading dimension that keeps them aligned
  const bool va = (a.lda & 3) == 0, vb = (a.ldb & 3) == 0;

  // loader of A (128 x 16 slice): stored [M][K]: thread -> rows tid/4 (+64),
  // k quad (tid&3)*4; stored [K][M]: k rows tid/32 (+8), m quad (tid&31)*4
  auto load_a = [&](const float *A, int k0, int h) -> float4 {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!AT) {
      const int m = m0 + (tid >> 2) + 64 * h, kk = k0 + (tid & 3) * 4;
      if (m >= Mx) return v;
      const float *p = A + (size_t)m * a.lda + kk;
      if (va && kk + 3 < kend) return __ldg(reinterpret_cast<const float4 *>(p));
      v.x = kk + 0 < kend ? __ldg(p + 0) : 0.f;
      v.y = kk + 1 < kend ? __ldg(p + 1) : 0.f;
      v.z = kk + 2 < kend ? __ldg(p + 2) : 0.f;
      v.w = kk + 3 < kend ? __ldg(p + 3) : 0.f;
    } else {
      const int kk = k0 + (tid >> 5) + 8 * h, m = m0 + (tid & 31) * 4;
      if (kk >= kend) return v;
      const float *p = A + (size_t)(GR && arow ? __ldg(arow + kk) : kk) * a.lda + m;
      if (va && m + 3 < Mx) return __ldg(reinterpret_cast<const float4 *>(p));
      v.x = m + 0 < Mx ? __ldg(p + 0) : 0.f;
      v.y = m + 1 < Mx ? __ldg(p + 1) : 0.f;
      v.z = m + 2 < Mx ? __ldg(p + 2) : 0.f;
      v.w = m + 3 < Mx ? __ldg(p + 3) : 0.f;
    }
    return v;
  };
  // loader of B (16 x 128 slice): stored [K][N]: k rows tid/32 (+8), n quad
  // (tid&31)*4; stored [N][K]: n rows tid/4 (+64), k quad (tid&3)*4
  auto load_b = [&](const float *B, int k0, int h) -> float4 {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!BT) {
      const int kk = k0 + (tid >> 5) + 8 * h, nn = n0 + (tid & 31) * 4;
      if (kk >= kend) return v;
      const float *p = B + (size_t)kk * a.ldb + nn;
      if (vb && nn + 3 < a.N) return __ldg(reinterpret_cast<const float4 *>(p));
      v.x = nn + 0 < a.N ? __ldg(p + 0) : 0.f;
      v.y = nn + 1 < a.N ? __ldg(p + 1) : 0.f;
      v.z = nn + 2 < a.N ? __ldg(p + 2) : 0.f;
      v.w = nn + 3 < a.N ? __ldg(p + 3) : 0.f;
    } else {
      const int nn = n0 + (tid >> 2) + 64 * h, kk = k0 + (tid & 3) * 4;
      if (nn >= a.N) return v;
      const float *p = B + (size_t)nn * a.ldb + kk;
      if (vb && kk + 3 < kend) return __ldg(reinterpret_cast<const float4 *>(p));
      v.x = kk + 0 < kend ? __ldg(p + 0) : 0.f;
      v.y = kk + 1 < kend ? __ldg(p + 1) : 0.f;
      v.z = kk + 2 < kend ? __ldg(p + 2) : 0.f;
      v.w = kk + 3 < kend ? __ldg(p + 3) : 0.f;
    }
    return v;
  };
  auto store = [&](int buf, const float4 (&av)[2], const float4 (&bv)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!AT) {
        const int r = (tid >> 2) + 64 * h, q = (tid & 3) * 4;
        As[buf][q + 0][r] = av[h].x;
        As[buf][q + 1][r] = av[h].y;
        As[buf][q + 2][r] = av[h].z;
        As[buf][q + 3][r] = av[h].w;
      } else {
        *reinterpret_cast<float4 *>(&As[buf][(tid >> 5) + 8 * h][(tid & 31) * 4]) = av[h];
      }
      if (!BT) {
        *reinterpret_cast<float4 *>(&Bs[buf][(tid >> 5) + 8 * h][(tid & 31) * 4]) = bv[h];
      } else {
        const int r = (tid >> 2) + 64 * h, q = (tid & 3) * 4;
        Bs[buf][q + 0][r] = bv[h].x;
        Bs[buf][q + 1][r] = bv[h].y;
        Bs[buf][q + 2][r] = bv[h].z;
        Bs[buf][q + 3][r] = bv[h].w;
      }
    }
  };

  // accumulator pairs: acc2[i][j] holds columns 2j, 2j+1 of row i (packed
  // FMAs, see fma2.cuh)
  unsigned long long acc2[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc2[i][j] = 0ull;

  // the pairs whose products are summed: pair 1 only with ksum
  const int npair = a.ksum ? 2 : 1;
  for (int p = 0; p < npair; ++p) {
    const int pi = a.ksum ? p : prob;
    // (selected, not indexed: a runtime index would copy the arguments to local memory)
    const float *A = (pi ? a.A[1] : a.A[0]) + offA, *B = (pi ? a.B[1] : a.B[0]) + offB;
    if (kbeg >= kend) break;
    float4 av[2] = {load_a(A, kbeg, 0), load_a(A, kbeg, 1)};
    float4 bv[2] = {load_b(B, kbeg, 0), load_b(B, kbeg, 1)};
    __syncthreads();  // the previous pair's last slice has been read
    store(0, av, bv);
    __syncthreads();
    int buf = 0;
    for (int k0 = kbeg; k0 < kend; k0 += BK) {
      const bool more = k0 + BK < kend;
      if (more) {  // the next slice into registers while this one is used
        av[0] = load_a(A, k0 + BK, 0);
        av[1] = load_a(A, k0 + BK, 1);
        bv[0] = load_b(B, k0 + BK, 0);
        bv[1] = load_b(B, k0 + BK, 1);
      }
      // the fragments of step kk + 1 are read while step kk's FMAs run
      float4 fa0[2], fa1[2], fb0[2], fb1[2];
      fa0[0] = *reinterpret_cast<const float4 *>(&As[buf][0][ty * 4]);
      fa1[0] = *reinterpret_cast<const float4 *>(&As[buf][0][64 + ty * 4]);
      fb0[0] = *reinterpret_cast<const float4 *>(&Bs[buf][0][tx * 4]);
      fb1[0] = *reinterpret_cast<const float4 *>(&Bs[buf][0][64 + tx * 4]);
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        const int cur = kk & 1, nxt = cur ^ 1;
        if (kk + 1 < BK) {
          fa0[nxt] = *reinterpret_cast<const float4 *>(&As[buf][kk + 1][ty * 4]);
          fa1[nxt] = *reinterpret_cast<const float4 *>(&As[buf][kk + 1][64 + ty * 4]);
          fb0[nxt] = *reinterpret_cast<const float4 *>(&Bs[buf][kk + 1][tx * 4]);
          fb1[nxt] = *reinterpret_cast<const float4 *>(&Bs[buf][kk + 1][64 + tx * 4]);
        }
        const float av8[8] = {fa0[cur].x, fa0[cur].y, fa0[cur].z, fa0[cur].w,
                              fa1[cur].x, fa1[cur].y, fa1[cur].z, fa1[cur].w};
        unsigned long long bp[4];
        bp[0] = pack2(fb0[cur].x, fb0[cur].y);
        bp[1] = pack2(fb0[cur].z, fb0[cur].w);
        bp[2] = pack2(fb1[cur].x, fb1[cur].y);
        bp[3] = pack2(fb1[cur].z, fb1[cur].w);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const unsigned long long ap = pack2(av8[i], av8[i]);
#pragma unroll
          for (int j = 0; j < 4; ++j) fma2(acc2[i][j], ap, bp[j]);
        }
      }
      if (more) {
        store(buf ^ 1, av, bv);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack2(acc2[i][j], acc[i][2 * j], acc[i][2 * j + 1]);

  // output rows ty*4+i (i<4) and 64+ty*4+i-4, columns tx*4+j and 64+tx*4+j-4
  float *const C = (prob ? a.C[1] : a.C[0]) + offC;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (m >= Mx) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int nn = n0 + h * 64 + tx * 4;
      const float4 v = make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2],
                                   acc[i][4 * h + 3]);
      if (a.part) {
        float *dst = a.part + (((size_t)prob * splits + split) * a.M + m) * a.N + nn;
        if ((a.N & 3) == 0 && nn + 3 < a.N) {
          *reinterpret_cast<float4 *>(dst) = v;
        } else {
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (nn + j < a.N) dst[j] = vv[j];
        }
      } else {
        float *dst = C + (size_t)m * a.ldc + nn;
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (nn + j < a.N) dst[j] = a.accumulate ? dst[j] + vv[j] : vv[j];
      }
    }
  }
}

// C_p = sum over the splits of problem p in order (+ C_p)
__global__ void __launch_bounds__(256) split_sum_kernel(const float *__restrict__ part, int splits,
                                                        int M, int N, float *C0, float *C1,
                                                        int ldc, int accumulate) {
  const size_t MN = (size_t)M * N;
  const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x;
  const int prob = blockIdx.y;
  if (i >= MN) return;
  const float *pp = part + (size_t)prob * splits * MN;
  float s = 0.f;
  for (int z = 0; z < splits; ++z) s += pp[(size_t)z * MN + i];
  const int m = (int)(i / N), nn = (int)(i % N);
  float *c = (prob ? C1 : C0) + (size_t)m * ldc + nn;
  *c = accumulate ? *c + s : s;
}

}  // namespace

int sgemm_splits(int M, int N, int K, int nprob) {
  const int tiles = (int)(ceil_div(M, BM) * ceil_div(N, BN)) * (nprob > 1 ? nprob : 1);
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
  if (b.nprob < 1) b.nprob = 1;
  if (b.ksum) b.nprob = 1;
  if (b.splits <= 1 || b.seg_off) b.part = nullptr;
  const int splits = b.part ? b.splits : 1;
  dim3 grid((unsigned)ceil_div(a.N, BN), (unsigned)ceil_div(a.M, BM), (unsigned)(splits * b.nprob));
  if (b.seg_off) {
    if (b.G <= 0) return MOE_OK;
    if (b.seg_k) grid.z = (unsigned)(b.G * b.nprob);
    else grid.y = (unsigned)b.mblk_upper;  // M = the rows of each group
  }
  const char *name = a.name ? a.name : "gate_grad_gemm";
  int rc;
  if (b.seg_off) {  // the two grouped shapes in use: K-grouped x^T D and M-grouped D W^T
    if (a.at && !a.bt) rc = launch(name, sgemm_kernel<true, false, true>, grid, dim3(NT), 0, st, b);
    else if (!a.at && a.bt) rc = launch(name, sgemm_kernel<false, true, true>, grid, dim3(NT), 0, st, b);
    else return MOE_EINVAL;
  } else if (!a.at && !a.bt) {
    rc = launch(name, sgemm_kernel<false, false, false>, grid, dim3(NT), 0, st, b);
  } else if (a.at && !a.bt) {
    rc = launch(name, sgemm_kernel<true, false, false>, grid, dim3(NT), 0, st, b);
  } else if (!a.at && a.bt) {
    rc = launch(name, sgemm_kernel<false, true, false>, grid, dim3(NT), 0, st, b);
  } else {
    rc = launch(name, sgemm_kernel<true, true, false>, grid, dim3(NT), 0, st, b);
  }
  if (rc != MOE_OK || !b.part) return rc;
  const size_t total = (size_t)a.M * a.N;
  return launch("gate_grad_split_sum", split_sum_kernel,
                dim3((unsigned)ceil_div((int64_t)total, 256), (unsigned)b.nprob), dim3(256), 0, st,
                (const float *)b.part, splits, a.M, a.N, b.C[0], b.C[b.nprob > 1 ? 1 : 0], a.ldc,
                a.accumulate);
}

}  // namespace moe
