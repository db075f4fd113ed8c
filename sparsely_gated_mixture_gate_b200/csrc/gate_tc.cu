// gate_tc.cu -- the gate's two projections on the tcgen05 tensor cores with
// fp32-level accuracy (three-pass TF32 split).
//
//   c = x W_g (+ b_g),  s = Softplus(x W_noise)     ([SGMoE-xyz] "Noisy Top-K 門控")
//
// [SGMoE-note] "缺点与局限性": the gate must be fp32 (bf16 diverged).  Every
// fp32 operand v is split as hi = v rounded to the nearest tf32 (10 mantissa
// bits), lo = v - hi (exact in fp32).  Then
//   x.W = hi_x.hi_W + hi_x.lo_W + lo_x.hi_W  (+ lo_x.lo_W, dropped)
// with each product taken by tcgen05.mma kind::tf32.  hi.hi is exact; the
// tensor core reads lo with at most 2^-10 of its own size lost (<= 2^-21 of
// v) and the dropped term is below 2^-22 of the product.  The tensor core's
// own fp32 accumulation does not round to nearest, so a long chain of MMAs
// into one accumulator drifts (measured: ~1e-5 on |x W| ~ 1 over K = 512).
// The chain is therefore cut every KC = 64 of K: the MMAs of one K-chunk
// accumulate into one of four tensor-memory buffers, the epilogue warps add
// the chunk into fp32 registers (round to nearest) while the MMAs fill the
// next ones.  Each chain is 24 MMAs long, and the result has about the
// accuracy of an fp32 multiply-add loop.
//
// Structure (same as the expert GEMM): persistent, one CTA per SM, 320
// threads.  Warp 0: TMA loads of x_hi, x_lo (128 rows x 32 fp32) and W_hi,
// W_lo (128 output columns x 32 fp32), 128-byte swizzle, 3 stages of 64 KiB.
// Warp 1: three MMAs (M=128, N=128, K=8) per 8-wide K step into one of the
// 128-column chunk buffers (four of them).  Warps 2-9: per chunk tcgen05.ld + fp32 adds into
// registers; per tile + b_g for the W_g columns or Softplus for the W_noise
// columns, fp32 stores of the valid rows.  Tiles
// are (group, M-block, N-block) with the N-block fastest so the CTAs that
// share an x tile run together.  The W operand is the transposed,
// concatenated [W_g | W_noise] of each group, K-major, prepared (with the
// hi/lo split of x) by two small kernels in this file.  No cluster multicast.
#include "tc_common.cuh"

namespace moe {
namespace {
using namespace tc;

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3;
constexpr int KB_PER_CHUNK = 2;               // K-chunk = 64: MMA chain length 2*4*3 = 24
constexpr int TILE_BYTES = 128 * 128;         // 128 rows x 128 bytes
constexpr int STAGE_BYTES = 4 * TILE_BYTES;   // x_hi, x_lo, W_hi, W_lo
constexpr int NUM_EPI = 256;
constexpr int NUM_THREADS = 64 + NUM_EPI;
constexpr int NBUF = 4;                       // K-chunk accumulators in tensor memory
constexpr uint32_t TMEM_COLS = NBUF * BN;     // all 512 columns
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr unsigned long long kWaitNs = 2000000000ull;
// kind::tf32: D fp32 (bits 4-5 = 1), A and B tf32 (format 2 at bits 7-9 and
// 10-12), both K-major, N>>3 at bits 17-22, M>>4 at bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

struct GateTcArgs {
  const int *seg_off;   // [G+1] or nullptr (one group of R rows)
  const int *seg_mblk;  // [G+1] exclusive scan of ceil(rows_g / BM), or nullptr
  int G, R, N, nb, K, nblk, mblk_flat;
  const float *bias;    // [G][nb] or nullptr
  float *c, *s;         // [R][nb]
  int *status;
};

__device__ __forceinline__ void decode(const GateTcArgs &a, int tile, int &g, int &row0,
                                       int &row_end, int &nbk) {
  const int v = tile / a.nblk;
  nbk = tile - v * a.nblk;
  if (a.seg_mblk) {
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.seg_mblk + mid) <= v) lo = mid; else hi = mid - 1;
    }
    g = lo;
    row0 = __ldg(a.seg_off + g) + (v - __ldg(a.seg_mblk + g)) * BM;
    row_end = __ldg(a.seg_off + g + 1);
  } else {
    g = 0;
    row0 = v * BM;
    row_end = a.R;
  }
}

__device__ __forceinline__ float softplus_f(float z) {
  return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gate_tf32x3_kernel(const __grid_constant__ CUtensorMap tmAhi,
                       const __grid_constant__ CUtensorMap tmAlo,
                       const __grid_constant__ CUtensorMap tmBhi,
                       const __grid_constant__ CUtensorMap tmBlo, GateTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NBUF + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull = [&](int c) { return bar0 + 8u * (2 * STAGES + c); };
  auto tempty = [&](int c) { return bar0 + 8u * (2 * STAGES + NBUF + c); };
  const uint32_t drain = bar0 + 8u * (2 * STAGES + 2 * NBUF);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int c = 0; c < NBUF; ++c) {
      mbar_init(tfull(c), 1);
      mbar_init(tempty(c), NUM_EPI);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = (a.seg_mblk ? __ldg(a.seg_mblk + a.G) : a.mblk_flat) * a.nblk;
  const int nkb = (a.K + BK - 1) / BK;
  bool failed = false;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int issued[STAGES];
    for (int s = 0; s < STAGES; ++s) issued[s] = -1;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      int g, row0, row_end, nbk;
      decode(a, tile, g, row0, row_end, nbk);
      const int brow = g * a.N + nbk * BN;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, kWaitNs)) { failed = true; break; }
        const uint32_t sa = sbase + stage * STAGE_BYTES;
        mbar_expect_tx(full(stage), STAGE_BYTES);
        tma_load_2d(sa, &tmAhi, full(stage), kb * BK, row0);
        tma_load_2d(sa + TILE_BYTES, &tmAlo, full(stage), kb * BK, row0);
        tma_load_2d(sa + 2 * TILE_BYTES, &tmBhi, full(stage), kb * BK, brow);
        tma_load_2d(sa + 3 * TILE_BYTES, &tmBlo, full(stage), kb * BK, brow);
        issued[stage] = (int)phase;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] >= 0) mbar_wait(full(s), (uint32_t)issued[s], nullptr, 100000000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    int stage = 0, buf = 0;
    uint32_t phase = 0, buf_phase = 0;
    bool issued_any = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      for (int kb0 = 0; kb0 < nkb && !failed; kb0 += KB_PER_CHUNK) {
        // a fresh chain for every K-chunk, in the buffer the epilogue drained
        if (!mbar_wait(tempty(buf), buf_phase ^ 1u, abort_flag, kWaitNs)) { failed = true; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        const int kb1 = min(nkb, kb0 + KB_PER_CHUNK);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full(stage), phase, abort_flag, kWaitNs)) { failed = true; break; }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {  // K = 8 tf32 = 32 bytes per MMA
            const uint64_t ahi = sw128_desc(sa + kk * 32);
            const uint64_t alo = sw128_desc(sa + TILE_BYTES + kk * 32);
            const uint64_t bhi = sw128_desc(sa + 2 * TILE_BYTES + kk * 32);
            const uint64_t blo = sw128_desc(sa + 3 * TILE_BYTES + kk * 32);
            tc_mma_tf32(d_tmem, ahi, bhi, IDESC, (kb != kb0 || kk != 0) ? 1u : 0u);
            tc_mma_tf32(d_tmem, ahi, blo, IDESC, 1u);
            tc_mma_tf32(d_tmem, alo, bhi, IDESC, 1u);
          }
          issued_any = true;
          tc_commit(empty(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (failed) break;
        tc_commit(tfull(buf));
        if (++buf == NBUF) { buf = 0; buf_phase ^= 1u; }
      }
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      if (issued_any) {
        tc_commit(drain);
        mbar_wait(drain, 0u, nullptr, 100000000ull);
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lanes 32q .. 32q+31
    const int half = (warp - 2) >> 2;    // tile columns [64*half, 64*half + 64)
    const bool vec = (a.nb & 3) == 0;
    int buf = 0;
    uint32_t buf_phase = 0;
    bool bad = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      int g, row0, row_end, nbk;
      decode(a, tile, g, row0, row_end, nbk);
      const int col0 = nbk * BN + half * 64;  // first output column of this warp
      float breg[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int col = col0 + u * 32 + lane;
        breg[u] = (a.bias && col < a.nb) ? __ldg(a.bias + (size_t)g * a.nb + col) : 0.f;
      }
      const int row = row0 + q * 32 + lane;
      const bool row_ok = row < row_end;
      float o[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) o[j] = 0.f;
      for (int kb0 = 0; kb0 < nkb; kb0 += KB_PER_CHUNK) {
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait(tfull(buf), buf_phase, abort_flag, kWaitNs));
        if (!ok) { failed = true; break; }
        tc_fence_after();
        uint32_t v[64];
        tmem_ld64(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + half * 64), v);
        tc_fence_before();
        mbar_arrive(tempty(buf));
        if (++buf == NBUF) { buf = 0; buf_phase ^= 1u; }
#pragma unroll
        for (int j = 0; j < 64; ++j) o[j] += __uint_as_float(v[j]);  // fp32, round to nearest
      }
      if (failed) break;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float b = __shfl_sync(0xffffffffu, breg[j >> 5], j & 31);
        const int col = col0 + j;
        o[j] = (col < a.nb) ? o[j] + b : softplus_f(o[j]);
      }
      if (row_ok) {
        const bool all_c = col0 + 64 <= a.nb;
        const bool all_s = col0 >= a.nb && col0 + 64 <= a.N;
        if (vec && (all_c || all_s)) {
          float *dst = all_c ? a.c + (size_t)row * a.nb + col0 : a.s + (size_t)row * a.nb + (col0 - a.nb);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            bad |= !isfinite(o[4 * u]) || !isfinite(o[4 * u + 1]) || !isfinite(o[4 * u + 2]) ||
                   !isfinite(o[4 * u + 3]);
            reinterpret_cast<float4 *>(dst)[u] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const int col = col0 + j;
            if (col < a.N) {
              bad |= !isfinite(o[j]);
              if (col < a.nb) a.c[(size_t)row * a.nb + col] = o[j];
              else a.s[(size_t)row * a.nb + (col - a.nb)] = o[j];
            }
          }
        }
      }
    }
    if (failed) *abort_flag = 1;
    if (bad && a.status) atomicOr(a.status, MOE_STATUS_NONFINITE);
  }

  if (failed && a.status) atomicOr(a.status, MOE_STATUS_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- operand preparation
// nearest tf32 (ties to even): keep sign, exponent and the top 10 mantissa bits
__device__ __forceinline__ float tf32_rne(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u & 0x7f800000u) == 0x7f800000u) return v;  // Inf / NaN unchanged
  u += 0x00000FFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// hi/lo split of the x rows (gathered through row_token for the grouped
// secondary gates): [R][d] each.
__global__ void split_rows_kernel(const float *x, const int *row_token, int R, int d, float *hi,
                                  float *lo) {
  const int q4 = d >> 2;
  const int64_t total = (int64_t)R * q4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / q4), q = (int)(i - (int64_t)r * q4);
    const int tok = row_token ? row_token[r] : r;
    const float4 v = __ldg(reinterpret_cast<const float4 *>(x + (size_t)tok * d) + q);
    const float4 h = make_float4(tf32_rne(v.x), tf32_rne(v.y), tf32_rne(v.z), tf32_rne(v.w));
    reinterpret_cast<float4 *>(hi)[i] = h;
    reinterpret_cast<float4 *>(lo)[i] = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
  }
}

// [W_g | W_noise] of every group, transposed to K-major and split:
// out[g][j][k] = (j < nb ? W_g[g][k][j] : W_noise[g][k][j - nb]), j < N.
__global__ void split_transpose_kernel(const float *Wg, const float *Wn, int d, int nb, int N,
                                       float *hi, float *lo) {
  __shared__ float t[32][33];
  const int g = blockIdx.z;
  const int k0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  const float *wg = Wg + (size_t)g * d * nb;
  const float *wn = Wn ? Wn + (size_t)g * d * nb : nullptr;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, j = j0 + threadIdx.x;
    float v = 0.f;
    if (k < d && j < N) v = j < nb ? wg[(size_t)k * nb + j] : wn[(size_t)k * nb + (j - nb)];
    t[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int j = j0 + i, k = k0 + threadIdx.x;
    if (j < N && k < d) {
      const float v = t[threadIdx.x][i];
      const float h = tf32_rne(v);
      const size_t o = ((size_t)g * N + j) * d + k;
      hi[o] = h;
      lo[o] = v - h;
    }
  }
}

}  // namespace

int launch_gate_tf32x3(const GateGemmArgs &a, int mblk_upper, float *xhi, float *xlo, float *whi,
                       float *wlo, cudaStream_t st) {
  const int N = a.nb * (a.noise ? 2 : 1);
  // operands: hi/lo of the (gathered) x rows and of the transposed weights
  {
    const int64_t total = (int64_t)a.R * (a.d / 4);
    const int grid = (int)std::min<int64_t>(ceil_div(total, 256), (int64_t)num_sms() * 8);
    MOE_TRY(launch("gate_split_x", split_rows_kernel, dim3(grid > 0 ? grid : 1), dim3(256), 0, st,
                   a.x, a.row_token, a.R, a.d, xhi, xlo));
    dim3 g3((unsigned)ceil_div(a.d, 32), (unsigned)ceil_div(N, 32), (unsigned)a.G);
    MOE_TRY(launch("gate_split_w", split_transpose_kernel, g3, dim3(32, 8), 0, st, a.Wg,
                   a.noise ? a.Wn : nullptr, a.d, a.nb, N, whi, wlo));
  }
  CUtensorMap ahi, alo, bhi, blo;
  MOE_TRY(make_map_2d(&ahi, xhi, 4, (uint64_t)a.d, (uint64_t)a.R, BM));
  MOE_TRY(make_map_2d(&alo, xlo, 4, (uint64_t)a.d, (uint64_t)a.R, BM));
  MOE_TRY(make_map_2d(&bhi, whi, 4, (uint64_t)a.d, (uint64_t)a.G * N, BN));
  MOE_TRY(make_map_2d(&blo, wlo, 4, (uint64_t)a.d, (uint64_t)a.G * N, BN));
  GateTcArgs t;
  t.seg_off = a.seg_off;
  t.seg_mblk = a.seg_mblk;
  t.G = a.G;
  t.R = a.R;
  t.N = N;
  t.nb = a.nb;
  t.K = a.d;
  t.nblk = (N + BN - 1) / BN;
  t.mblk_flat = (int)ceil_div(a.R, BM);
  t.bias = a.bias;
  t.c = a.c;
  t.s = a.s;
  t.status = a.status;
  const int64_t upper = (int64_t)mblk_upper * t.nblk;
  const int grid = (int)std::min<int64_t>(upper, num_sms());
  static PerDevice attrs;
  MOE_TRY(attrs.get([](int, int *) {
    return cudaFuncSetAttribute(gate_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES) == cudaSuccess
               ? MOE_OK
               : MOE_ECUDA;
  }));
  if (grid <= 0) return MOE_OK;
  return launch("gate_gemm_tf32x3", gate_tf32x3_kernel, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, st,
                ahi, alo, bhi, blo, t);
}

}  // namespace moe
