// gate_gemm.cu -- the gate's two projections in fp32:
//   c = x W_g (+ b_g)          (clean logits)
//   s = Softplus(x W_noise)    (noise scale)
// [SGMoE-xyz] "Noisy Top-K 門控": H(x)_i = (x W_g)_i + StandardNormal() *
// Softplus((x W_noise)_i); [SGMoE-note] "缺点与局限性": the gate needs fp32
// (bf16 made training diverge), so this contraction stays on the FP32 pipes.
//
// One kernel serves the flat gate, the primary gate and the grouped
// secondary gates of the hierarchical layer: rows can be gathered from x
// through row_token, and rows are split into groups (ragged M) that each use
// their own weights.  The N dimension runs over the columns of W_g followed
// by those of W_noise (2 nb columns with noise), tiled in 128-column pieces
// (blockIdx.y), so one launch computes both c and s and a narrow gate (the
// hierarchical layer's primary gate has nb = 64) fills whole tiles.
//
// Tile: 128 x 128 x 16, 256 threads, 8x8 outputs per thread held as two 4x4
// quadrants (rows ty*4, 64+ty*4; cols tx*4, 64+tx*4) so the shared-memory
// reads of a warp are broadcast / conflict free.  Double-buffered shared
// memory, global loads of the next K-slice overlap the FMAs of the current,
// and the register fragments of the next k step are read during the FMAs of
// this one.  The multiply-adds are packed (fma.rn.f32x2: two independent
// fp32 FMAs, each rounded as fmaf would): the accumulators of columns j, j+1
// form a pair, multiplied by the pair (a_i, a_i) and the pair (b_j, b_j+1),
// so one instruction does two of the 64 per k step and the FMA issue slots
// halve; every output is still one fmaf chain over k in order.
#include "fma2.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = kGateBM, BN = kGateBN, BK = 16, NT = 256;
constexpr int APAD = 4;  // As row padding (keeps 16-byte alignment)

__device__ __forceinline__ float softplus_f(float z) {
  return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
}

__global__ void __launch_bounds__(NT, 2) gate_gemm_kernel(GateGemmArgs a) {
  __shared__ __align__(16) float As[2][BK][BM + APAD];
  __shared__ __align__(16) float Bs[2][BK][BN];

  // ---- which group, which rows
  const int mblk = blockIdx.x;
  int g = 0, row0, row_end;
  if (a.seg_mblk) {
    const int total = a.seg_mblk[a.G];
    if (mblk >= total) return;
    int lo = 0, hi = a.G - 1;  // largest g with seg_mblk[g] <= mblk
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.seg_mblk[mid] <= mblk) lo = mid; else hi = mid - 1;
    }
    g = lo;
    row0 = a.seg_off[g] + (mblk - a.seg_mblk[g]) * BM;
    row_end = a.seg_off[g + 1];
  } else {
    row0 = mblk * BM;
    row_end = a.R;
    if (row0 >= row_end) return;
  }
  const int nb = a.nb;
  const int ncol = a.noise ? 2 * nb : nb;      // columns of [W_g | W_noise]
  const int col0 = blockIdx.y * BN;            // first column of this tile
  const float *Bg = a.Wg + (size_t)g * a.d * nb;
  const float *Bn = a.noise ? a.Wn + (size_t)g * a.d * nb : nullptr;
  const bool vecB = (nb & 3) == 0;             // a column quad never straddles the two

  const int tid = threadIdx.x;
  // A loader: rows ar and ar + 64 (ar = tid/4), k quad aq = (tid&3)*4
  const int ar = tid >> 2, aq = (tid & 3) * 4;
  const float *Arow[2] = {nullptr, nullptr};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int arow = row0 + ar + 64 * h;
    if (arow < row_end) {
      const int tok = a.row_token ? a.row_token[arow] : arow;
      Arow[h] = a.x + (size_t)tok * a.d;
    }
  }
  // B loader: k rows bk and bk + 8 (bk = tid/32), col quad bc = (tid&31)*4
  const int bk = tid >> 5, bc = (tid & 31) * 4;
  const int bcol = col0 + bc;

  auto load_a = [&](int k0, int h) -> float4 {
    if (!Arow[h]) return make_float4(0.f, 0.f, 0.f, 0.f);
    // d is a multiple of 8: a K tail inside a 16-wide slice reads zeros
    if (k0 + aq >= a.d) return make_float4(0.f, 0.f, 0.f, 0.f);
    return __ldg(reinterpret_cast<const float4 *>(Arow[h] + k0 + aq));
  };
  // element (kr, column vc) of [W_g | W_noise]
  auto b_elem = [&](int kr, int vc) -> float {
    if (vc >= ncol) return 0.f;
    return vc < nb ? __ldg(Bg + (size_t)kr * nb + vc) : __ldg(Bn + (size_t)kr * nb + (vc - nb));
  };
  auto load_b = [&](int k0, int h) -> float4 {
    const int kr = k0 + bk + 8 * h;
    if (kr >= a.d) return make_float4(0.f, 0.f, 0.f, 0.f);
    if (vecB && bcol + 3 < ncol) {
      const float *p = bcol < nb ? Bg + (size_t)kr * nb + bcol : Bn + (size_t)kr * nb + (bcol - nb);
      return __ldg(reinterpret_cast<const float4 *>(p));
    }
    return make_float4(b_elem(kr, bcol), b_elem(kr, bcol + 1), b_elem(kr, bcol + 2),
                       b_elem(kr, bcol + 3));
  };
  auto store_tiles = [&](int buf, const float4 (&av)[2], const float4 (&bv)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      As[buf][aq + 0][ar + 64 * h] = av[h].x;
      As[buf][aq + 1][ar + 64 * h] = av[h].y;
      As[buf][aq + 2][ar + 64 * h] = av[h].z;
      As[buf][aq + 3][ar + 64 * h] = av[h].w;
      *reinterpret_cast<float4 *>(&Bs[buf][bk + 8 * h][bc]) = bv[h];
    }
  };

  // accumulator pairs: acc2[i][j] holds columns 2j, 2j+1 of row i
  unsigned long long acc2[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc2[i][j] = 0ull;

  const int tx = tid & 15, ty = tid >> 4;
  const int nk = (a.d + BK - 1) / BK;
  float4 av[2] = {load_a(0, 0), load_a(0, 1)}, bv[2] = {load_b(0, 0), load_b(0, 1)};
  store_tiles(0, av, bv);
  __syncthreads();

  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        av[h] = load_a((kt + 1) * BK, h);
        bv[h] = load_b((kt + 1) * BK, h);
      }
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
      const float ar_[8] = {fa0[cur].x, fa0[cur].y, fa0[cur].z, fa0[cur].w,
                            fa1[cur].x, fa1[cur].y, fa1[cur].z, fa1[cur].w};
      unsigned long long bp[4];
      bp[0] = pack2(fb0[cur].x, fb0[cur].y);
      bp[1] = pack2(fb0[cur].z, fb0[cur].w);
      bp[2] = pack2(fb1[cur].x, fb1[cur].y);
      bp[3] = pack2(fb1[cur].z, fb1[cur].w);
      unsigned long long ap[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ap[i] = pack2(ar_[i], ar_[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j)  // each B pair over the eight rows (measured 1% faster)
#pragma unroll
        for (int i = 0; i < 8; ++i) fma2(acc2[i][j], ap[i], bp[j]);
    }
    if (kt + 1 < nk) {
      store_tiles(buf ^ 1, av, bv);
    }
    __syncthreads();
  }

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack2(acc2[i][j], acc[i][2 * j], acc[i][2 * j + 1]);

  // ---- epilogue: columns [0, nb) are c (+ bias), [nb, 2 nb) are s = Softplus
  const float *bias = a.bias ? a.bias + (size_t)g * nb : nullptr;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = row0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (row >= row_end) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = col0 + h * 64 + tx * 4;
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float z = acc[i][h * 4 + j];
        const int vc = col + j;
        if (vc < nb) {
          if (bias) z += bias[vc];
          bad |= !isfinite(z);
        } else if (vc < ncol) {
          z = softplus_f(z);
          bad |= !isfinite(z);
        }
        v[j] = z;
      }
      if (vecB && col + 3 < ncol) {
        float *dst = col < nb ? a.c + (size_t)row * nb + col : a.s + (size_t)row * nb + (col - nb);
        *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int vc = col + j;
          if (vc < nb) a.c[(size_t)row * nb + vc] = v[j];
          else if (vc < ncol) a.s[(size_t)row * nb + (vc - nb)] = v[j];
        }
      }
    }
  }
  if (bad && a.status) atomicOr(a.status, MOE_STATUS_NONFINITE);
}

}  // namespace

int launch_gate_gemm(const GateGemmArgs &a, int mblk_upper, cudaStream_t st) {
  const int ncol = a.noise ? 2 * a.nb : a.nb;
  dim3 grid(mblk_upper, (ncol + BN - 1) / BN);
  return launch("gate_gemm_fp32", gate_gemm_kernel, grid, dim3(NT), 0, st, a);
}

}  // namespace moe
