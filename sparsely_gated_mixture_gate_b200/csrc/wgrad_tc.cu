// wgrad_tc.cu -- the experts' weight gradients on the tensor cores.
//
// With expert e's rows r = offsets[e] .. offsets[e+1]-1 (the dispatch's
// expert-contiguous order) the forward's y_e = hid_e W2_e^T + b2_e and
// hid_e = ReLU(x_e W1_e^T + b1_e) give
//   dW2_e = sum_r dy_perm[r]^T hid[r]    ([d][f], the layout of W2)
//   dW1_e = sum_r dhid[r]^T  x_perm[r]   ([f][d], the layout of W1)
// i.e. GEMMs whose K is the expert's row count (ragged) and whose operands
// are the row-major activations read MN-major.  The biases' gradients are
// plain column sums (backward.cu).
//
// One persistent kernel, one CTA per SM, 320 threads, the same roles as the
// forward's expert kernel:
//   warp 0  TMA producer: per stage the A tile (128 M x 32 rows, two 64-column
//           boxes) and the B tile (256 N x 32 rows, four boxes), 128-byte
//           swizzle, 8 stages.  32-row K steps: the hierarchical layer's
//           experts hold ~32 rows each, and 64-row steps loaded as many rows
//           of the next expert as of their own (measured: 32-row steps 6% and
//           4-9% faster than 64-row steps on the hierarchical layer and at 256
//           experts of ~128 rows; 16-row steps 6% slower on the latter)
//   warp 1  MMA: tcgen05.mma kind::f16 with both operands MN-major (M=128,
//           N=256, K=16).  The last K step of an expert reads rows that
//           belong to the next expert (or the zero fill past the end); the
//           warp zeroes those rows of both tiles in shared memory (at most
//           15 per tile, whole 128-byte rows so the swizzle does not matter),
//           fences them to the async proxy and skips the 16-row steps that
//           hold none of the expert's rows.
//   warps 2-9  epilogue: tcgen05.ld of the fp32 accumulator, staged through
//           4 KiB of shared memory per warp so that each store writes four
//           whole 128-byte row segments, streaming stores (the gradients are
//           not read again by this pass).  An expert without rows gets zeros.
// Tiles: expert-major (its rows stay in L2 for all of its tiles), dW2 tiles
// then dW1 tiles, M-block fastest.  Every wait is bounded (about two seconds
// of %globaltimer); a timeout sets MOE_STATUS_TIMEOUT and the CTA drains and
// returns.  No cluster multicast.
#include "tc_common.cuh"

namespace moe {
namespace {
using namespace tc;

constexpr int BM = 128, BN = 256, BK = 32, STAGES = 8;
constexpr int BOX = 64 * BK * 2;  // one 64-column x BK-row box, 4 KiB
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_EPI = 256;
constexpr int NUM_EPI_WARPS = NUM_EPI / 32;
constexpr int NUM_THREADS = 64 + NUM_EPI;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int BAR_BYTES = 256;
constexpr int EPI_STAGE_BYTES = 32 * 128;  // per epilogue warp: 32 rows x 32 fp32
constexpr int SMEM_BYTES =
    STAGES * STAGE_BYTES + 1024 + BAR_BYTES + NUM_EPI_WARPS * EPI_STAGE_BYTES;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
// full/empty per stage, tfull/tempty per accumulator, drain; then the TMEM slot and abort flag
static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
constexpr unsigned long long kWaitNs = 2000000000ull;

// kind::f16, D fp32, A and B bf16, both MN-major (bits 15, 16), N>>3, M>>4
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct WArgs {
  const int *offsets;
  int n, d, f;
  int mb0, nb0, mb1, nb1;  // M- and N-blocks of dW2 (M = d, N = f) and dW1 (M = f, N = d)
  float *dW2, *dW1;
  int *status;
};

struct TileInfo {
  int e, set, mb, nb, off, cnt;
};

__device__ __forceinline__ TileInfo tile_info(const WArgs &a, int tile) {
  const int t0 = a.mb0 * a.nb0, per = t0 + a.mb1 * a.nb1;
  TileInfo ti;
  ti.e = tile / per;
  int r = tile - ti.e * per;
  ti.set = r >= t0;
  if (ti.set) r -= t0;
  const int mb = ti.set ? a.mb1 : a.mb0;
  ti.nb = r / mb;
  ti.mb = r - ti.nb * mb;
  ti.off = __ldg(a.offsets + ti.e);
  ti.cnt = __ldg(a.offsets + ti.e + 1) - ti.off;
  return ti;
}

__device__ __forceinline__ void st_shared_zero16(uint32_t addr) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                 const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                 WArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES] empty[STAGES] tfull[2] tempty[2] drain[1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull = [&](int c) { return bar0 + 8u * (2 * STAGES + c); };
  auto tempty = [&](int c) { return bar0 + 8u * (2 * STAGES + 2 + c); };
  const uint32_t drain = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t sbase = smem_u32(smem);
  uint8_t *const stage_epi_all = smem + STAGES * STAGE_BYTES + BAR_BYTES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int c = 0; c < 2; ++c) {
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

  const int total = a.n * (a.mb0 * a.nb0 + a.mb1 * a.nb1);
  bool failed = false;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int issued[STAGES];
    for (int s = 0; s < STAGES; ++s) issued[s] = -1;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const TileInfo ti = tile_info(a, tile);
      const CUtensorMap *mA = ti.set ? &tmA1 : &tmA0;
      const CUtensorMap *mB = ti.set ? &tmB1 : &tmB0;
      const int nkb = (ti.cnt + BK - 1) / BK;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, kWaitNs)) { failed = true; break; }
        const uint32_t sa = sbase + stage * STAGE_BYTES;
        const int row = ti.off + kb * BK;
        mbar_expect_tx(full(stage), STAGE_BYTES);
#pragma unroll
        for (int i = 0; i < BM / 64; ++i)
          tma_load_2d(sa + i * BOX, mA, full(stage), ti.mb * BM + 64 * i, row);
#pragma unroll
        for (int i = 0; i < BN / 64; ++i)
          tma_load_2d(sa + A_BYTES + i * BOX, mB, full(stage), ti.nb * BN + 64 * i, row);
        issued[stage] = (int)phase;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] >= 0) mbar_wait(full(s), (uint32_t)issued[s], nullptr, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA (lane 0 issues; the warp zeroes tails)
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool issued_any = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const TileInfo ti = tile_info(a, tile);
      const int nkb = (ti.cnt + BK - 1) / BK;
      if (!__all_sync(0xffffffffu, mbar_wait(tempty(acc), acc_phase ^ 1u, abort_flag, kWaitNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(full(stage), phase, abort_flag, kWaitNs))) {
          failed = true;
          break;
        }
        const uint32_t sa = sbase + stage * STAGE_BYTES;
        const int valid = min(BK, ti.cnt - kb * BK);  // this expert's rows in the stage
        const int used = (valid + 15) & ~15;           // rows the MMAs read
        if (valid < used) {
          // rows valid .. used-1 belong to another expert: zero them in all six boxes
          const int nr = used - valid, per_box = nr * 8;
          for (int c = lane; c < 6 * per_box; c += 32) {
            const int b = c / per_box, rem = c - b * per_box;
            const int r = valid + (rem >> 3), ch = rem & 7;
            const uint32_t base = b < 2 ? sa + b * BOX : sa + A_BYTES + (b - 2) * BOX;
            st_shared_zero16(base + r * 128 + ch * 16);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          for (int kk = 0; kk < used / 16; ++kk)
            tc_mma_f16(d_tmem, sw128_mn_desc(sa + kk * 2048, BOX),
                       sw128_mn_desc(sa + A_BYTES + kk * 2048, BOX), IDESC, (kb | kk) != 0);
          tc_commit(empty(stage));
        }
        issued_any = true;
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (failed) break;
      if (lane == 0) tc_commit(tfull(acc));  // no MMAs (no rows): the epilogue writes zeros
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      if (issued_any && lane == 0) {
        tc_commit(drain);
        mbar_wait(drain, 0u, nullptr, 100000000ull);
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lanes 32q .. 32q+31
    const int half = (warp - 2) >> 2;    // columns [128*half, +128) of the tile
    uint8_t *const stage_epi = stage_epi_all + (warp - 2) * EPI_STAGE_BYTES;
    const int rr = lane >> 3, cc = lane & 7;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const TileInfo ti = tile_info(a, tile);
      const int M = ti.set ? a.f : a.d, N = ti.set ? a.d : a.f;
      float *const out = (ti.set ? a.dW1 : a.dW2) + (size_t)ti.e * M * N;
      const int m0 = ti.mb * BM + q * 32;  // this warp's first row
      const int rows_here = M - m0;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull(acc), acc_phase, abort_flag, kWaitNs));
      if (!ok) { failed = true; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int cl = half * 128 + c * 64;
        uint32_t v[64];
        if (ti.cnt > 0) {
          tmem_ld64(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + cl), v);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = 0u;
        }
        const int col0 = ti.nb * BN + cl;
        if (col0 < N && rows_here > 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // lane l's row, 32 columns: chunk u (4 floats) at slot u ^ (l & 7)
            uint8_t *row_st = stage_epi + lane * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4 *>(row_st + ((u ^ (lane & 7)) << 4)) =
                  make_uint4(v[32 * h + 4 * u], v[32 * h + 4 * u + 1], v[32 * h + 4 * u + 2],
                             v[32 * h + 4 * u + 3]);
            __syncwarp();
            const int cbase = col0 + 32 * h;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = i * 4 + rr;
              const uint4 w4 =
                  *reinterpret_cast<const uint4 *>(stage_epi + r * 128 + ((cc ^ (r & 7)) << 4));
              const int col = cbase + cc * 4;
              if (r < rows_here && col < N)
                __stcs(reinterpret_cast<float4 *>(out + (size_t)(m0 + r) * N + col),
                       make_float4(__uint_as_float(w4.x), __uint_as_float(w4.y),
                                   __uint_as_float(w4.z), __uint_as_float(w4.w)));
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (failed) *abort_flag = 1;
  }

  if (failed && a.status) atomicOr(a.status, MOE_STATUS_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

int launch_wgrad_bf16(const WgradArgs &a, cudaStream_t st) {
  if (a.n == 0) return MOE_OK;
  static PerDevice setup;  // the kernel's shared-memory attribute, then its resident CTAs
  int ctas = 0;
  MOE_TRY(setup.get([](int, int *out) {
    if (cudaFuncSetAttribute(wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return MOE_ECUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wgrad_kernel, NUM_THREADS,
                                                      SMEM_BYTES) != cudaSuccess ||
        per_sm < 1)
      return MOE_ECUDA;
    *out = per_sm * num_sms();
    return MOE_OK;
  }, &ctas));
  // rows beyond S read as zero; every box is 64 columns x BK rows
  const uint64_t S = (uint64_t)(a.S > 0 ? a.S : 1);
  CUtensorMap mA0, mB0, mA1, mB1;
  MOE_TRY(tc::make_map_2d(&mA0, a.dy_perm, 2, (uint64_t)a.d, S, BK));
  MOE_TRY(tc::make_map_2d(&mB0, a.hid, 2, (uint64_t)a.f, S, BK));
  MOE_TRY(tc::make_map_2d(&mA1, a.dhid, 2, (uint64_t)a.f, S, BK));
  MOE_TRY(tc::make_map_2d(&mB1, a.x_perm, 2, (uint64_t)a.d, S, BK));
  WArgs w;
  w.offsets = a.offsets;
  w.n = a.n;
  w.d = a.d;
  w.f = a.f;
  w.mb0 = (int)ceil_div(a.d, BM);
  w.nb0 = (int)ceil_div(a.f, BN);
  w.mb1 = (int)ceil_div(a.f, BM);
  w.nb1 = (int)ceil_div(a.d, BN);
  w.dW2 = a.dW2;
  w.dW1 = a.dW1;
  w.status = a.status;
  const int64_t total = (int64_t)a.n * (w.mb0 * w.nb0 + w.mb1 * w.nb1);
  const int grid = (int)(total < ctas ? total : ctas);
  return launch(a.name ? a.name : "wgrad_tcgen05", wgrad_kernel, dim3(grid), dim3(NUM_THREADS),
                (size_t)SMEM_BYTES, st, mA0, mB0, mA1, mB1, w);
}

}  // namespace moe
