// expert_tc.cu -- the experts' two dense contractions on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory, operands by TMA).
//
// [SGMoE-note] "Sparsely-Gated MoE 层架构": every expert is a feed-forward
// network with one ReLU hidden layer.  With the kept rows of expert e stored
// contiguously (rows offsets[e] .. offsets[e+1]-1 of x_perm):
//   GEMM1: hid    = ReLU(x_perm_e W1_e^T + b1_e)   (bf16 out)
//   GEMM2: y_perm = hid_e W2_e^T + b2_e            (bf16 out)
// Both are "grouped" GEMMs with a ragged M per expert and K-major operands.
// The backward pass's activation gradients have the same two-step shape:
//   GEMM1': dhid    = (dy_perm_e W2_e) * [hid > 0]  (bf16 out; ReLU mask)
//   GEMM2': dx_perm = dhid_e W1_e                   (bf16 out)
// with the same tiles (N = f, then N = d); their B operands are the weights
// as stored, i.e. MN-major (N contiguous), loaded as four 64-column boxes.
//
// One persistent kernel runs both, one CTA per SM, 320 threads.  The two
// GEMMs' tiles form one list (see tile_at): M-block by M-block, the GEMM1
// tiles of M-block s and then the GEMM2 tiles of M-block s - lag.  When the
// experts stream their weights at the HBM limit (few rows per expert) the
// lag is a few waves of tiles, so an M-block's rows of hid are read back by
// GEMM2 a few waves after they were written, from L2, instead of after the
// whole of GEMM1; otherwise the lag covers every M-block and all of GEMM1
// runs first (see kInterleaveMaxRows).  CTA i takes tiles i, i + grid, ...
// A GEMM2 tile of M-block m waits (bounded) until the epilogues of all GEMM1
// tiles of m have published their rows of hid (a counter per M-block, and one
// for all of GEMM1: once a CTA has seen all of GEMM1 published, its later
// GEMM2 tiles need no check).  Every GEMM1 tile of m comes before the GEMM2 tiles of m in
// the list, and every CTA runs its tiles in list order, so the unfinished
// tile earliest in the list never waits on a later one; the launch is
// cooperative, so every CTA is resident and no wait can depend on a CTA that
// has not started.
//   warp 0  TMA producer: 128x64 A tile + 256x64 B tile per stage (128-byte
//           swizzle), 4 stages, mbarrier transaction counts
//   warp 1  MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M=128,
//           N=256, K=16, four per stage; tcgen05.commit frees the stage
//   warps 2-9  epilogue: two warps per 32-lane quarter of tensor memory, one
//           per 128-column half; tcgen05.ld of the fp32 accumulator 64
//           columns at a time, bias (prefetched into registers before the
//           wait, broadcast by shuffles), ReLU, bf16; the warp's 32 x 64 block
//           goes through its own 4 KiB of shared memory (XOR-swizzled 16-byte
//           chunks) so that every store instruction writes four whole 128-byte
//           row segments, masked to the expert's valid rows; the hidden layer's
//           stores carry an evict-last L2 policy (GEMM2 reads it back)
// Two accumulators of 256 columns (all 512 TMEM columns) let the epilogue of
// one tile overlap the main loop of the next.  M-blocks are numbered expert by
// expert, so the M-blocks that share a weight tile run at about the same time
// and the weights stream from HBM once.
// No cluster multicast anywhere.
//
// Every wait is bounded (about two seconds of %globaltimer); a wait that runs
// out sets MOE_STATUS_TIMEOUT, raises an abort flag seen by the other roles,
// drains the copies and MMAs this CTA issued (again bounded), frees its
// tensor memory and returns.
#include <atomic>
#include <climits>

#include "tc_common.cuh"

namespace moe {
namespace {
using namespace tc;

constexpr int BM = kExpertBM, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_EPI = 256;                 // epilogue threads (warps 2-9)
constexpr int NUM_EPI_WARPS = NUM_EPI / 32;
constexpr int NUM_THREADS = 64 + NUM_EPI;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int BAR_BYTES = 256;
constexpr int EPI_STAGE_BYTES = 32 * 128;    // per epilogue warp: 32 rows x 64 bf16
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + BAR_BYTES + NUM_EPI_WARPS * EPI_STAGE_BYTES;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr unsigned long long kWaitNs = 2000000000ull;
// The lag of the interleaved schedule in waves of tiles (see tile_at): 3, or 4
// from kLag4Rows rows per expert on average (measured: 32 and 64 rows best at
// 3 waves, 128 rows 1.5-2.5% faster at 4 or 5 than at 3; 2 waves slower
// everywhere, GEMM2 tiles then waiting on GEMM1 tiles still in flight)
constexpr int kLagWaves = 3, kLag4Rows = 96;
// Interleave only while the experts average fewer rows than this: each byte of
// expert weights then feeds fewer FLOPs than about 0.75 x (bf16 tensor peak /
// HBM bandwidth), so the weights stream at the HBM limit and the hidden
// layer's DRAM round trip competes with them.  With more rows the GEMMs sit
// near the tensor-bound ridge, that round trip costs nothing HBM cannot
// spare, and interleaving measured 3-8% slower (switch-top1, 256 rows per
// expert) than running all of GEMM1 first.
constexpr int kInterleaveMaxRows = 192;

// instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9
// = 1), B bf16 (bits 10-12 = 1), both K-major (bits 15, 16 = 0), N>>3 at bits
// 17-22, M>>4 at bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_BMN = IDESC | (1u << 16);  // B MN-major (bit 16)
constexpr int BOX_MN = 64 * BK * 2;                  // one 64-column box of an MN-major tile

struct GemmArgs {
  const int4 *tiles;     // per tile: {expert, first row, valid rows, N-block | M-block << 8}
  int N, K, nblk;
  const float *bias;     // [n][N] or nullptr
  __nv_bfloat16 *D;      // [S][N]
  int relu;
  const __nv_bfloat16 *mask;  // [S][N] or nullptr: D = acc where mask > 0, else 0
};

struct FfnArgs {
  GemmArgs g[2];         // GEMM1, GEMM2
  const int *mprefix;    // [n+1]; mprefix[n] M-blocks
  int n;
  int *mdone;            // [M-blocks + 1] GEMM1 epilogue warps finished, per M-block; the
                         // last entry counts them over all of GEMM1
  int *status;
  unsigned long long xwait_ns;  // limit of a GEMM2 tile's wait for its M-block of hid
  int withhold_mblk;     // test hook: this M-block's GEMM1 tiles never publish (-1: none)
  int lag;               // M-blocks between a GEMM1 M-block and GEMM2's in the tile list
};

// Tile c of the list: the GEMM1 tiles of M-blocks 0 .. lag-1, then for s =
// lag, lag+1, ... the GEMM1 tiles of M-block s followed by the GEMM2 tiles of
// M-block s - lag, then the GEMM2 tiles of the last lag M-blocks.  The tile
// tables are M-block major (entry M-block * nblk + N-block).  Returns the
// GEMM (0, 1) and the entry of its table.
__device__ __forceinline__ int2 tile_at(int c, int mtotal, int n1, int n2, int lag) {
  const int lead = min(lag, mtotal);
  if (c < lead * n1) return make_int2(0, c);
  c -= lead * n1;
  const int w = n1 + n2, both = (mtotal - lead) * w;
  if (c < both) {
    const int s = c / w, r = c - s * w;
    return r < n1 ? make_int2(0, (lead + s) * n1 + r) : make_int2(1, s * n2 + (r - n1));
  }
  return make_int2(1, (mtotal - lead) * n2 + (c - both));
}

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// bounded wait until *p >= target (acquire at GPU scope)
__device__ __noinline__ bool wait_count(const int *p, int target, volatile int *abort_flag,
                                        unsigned long long limit_ns) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire(p) >= target) return true;
    if ((it & 15u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) return false;
    }
  }
}

// BMN: B operands MN-major (the backward pass's activation gradients)
template <bool BMN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    expert_ffn_kernel(const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmB1,
                      const __grid_constant__ CUtensorMap tmA2,
                      const __grid_constant__ CUtensorMap tmB2, FfnArgs a) {
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
  // epilogue warps' output staging, 4 KiB each, after the barriers
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

  const int mtotal = __ldg(a.mprefix + a.n);
  const int T1 = mtotal * a.g[0].nblk, total = T1 + mtotal * a.g[1].nblk;
  const int ready = NUM_EPI_WARPS * a.g[0].nblk;  // arrivals that complete an M-block of hid
  bool failed = false;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int issued[STAGES];
    for (int s = 0; s < STAGES; ++s) issued[s] = -1;
    bool g1_all = false;  // all of GEMM1's hid seen published (acquire + proxy fence done)
    auto entry = [&](int t) {
      if (t >= total) return make_int4(0, 0, 0, 0);
      const int2 w = tile_at(t, mtotal, a.g[0].nblk, a.g[1].nblk, a.lag);
      return __ldg(a.g[w.x].tiles + w.y);
    };
    int4 ti = entry(blockIdx.x);
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const int which = tile_at(tile, mtotal, a.g[0].nblk, a.g[1].nblk, a.lag).x;
      const GemmArgs &g = a.g[which];
      const int4 next = entry(tile + gridDim.x);  // fetched while this tile's loads go out
      if (which && !g1_all) {
        // hid rows of this M-block: every GEMM1 epilogue warp of it has
        // published them; then order the TMA reads after that observation
        if (ld_acquire(a.mdone + mtotal) >= NUM_EPI_WARPS * T1) {
          g1_all = true;
        } else if (!wait_count(a.mdone + (ti.w >> 8), ready, abort_flag, a.xwait_ns)) {
          failed = true;
          break;
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      const CUtensorMap *mA = which ? &tmA2 : &tmA1;
      const CUtensorMap *mB = which ? &tmB2 : &tmB1;
      const int nkb = (g.K + BK - 1) / BK;
      const int brow = ti.x * g.N + (ti.w & 0xFF) * BN;  // K-major B: first weight row
      const int bcol = (ti.w & 0xFF) * BN;                // MN-major B: first column
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, kWaitNs)) { failed = true; break; }
        const uint32_t sa = sbase + stage * STAGE_BYTES;
        mbar_expect_tx(full(stage), STAGE_BYTES);
        tma_load_2d(sa, mA, full(stage), kb * BK, ti.y);
        if (BMN) {
          // rows ti.x*K + kb*BK .. +63 of the [n*K][N] weights, four 64-column boxes
#pragma unroll
          for (int i = 0; i < BN / 64; ++i)
            tma_load_2d(sa + A_BYTES + i * BOX_MN, mB, full(stage), bcol + 64 * i,
                        ti.x * g.K + kb * BK);
        } else {
          tma_load_2d(sa + A_BYTES, mB, full(stage), kb * BK, brow);
        }
        issued[stage] = (int)phase;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      ti = next;
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      // let the copies this thread started land before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] >= 0) mbar_wait(full(s), (uint32_t)issued[s], nullptr, 100000000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool issued_any = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const int nkb = (a.g[tile_at(tile, mtotal, a.g[0].nblk, a.g[1].nblk, a.lag).x].K + BK - 1) / BK;
      if (!mbar_wait(tempty(acc), acc_phase ^ 1u, abort_flag, kWaitNs)) { failed = true; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(full(stage), phase, abort_flag, kWaitNs)) { failed = true; break; }
        tc_fence_after();
        const uint32_t sa = sbase + stage * STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // K-major: the 16-wide K step is 32 bytes into each 128-byte row;
          // MN-major: 16 rows of 128 bytes further on
          const uint64_t bdesc = BMN ? sw128_mn_desc(sa + A_BYTES + kk * 2048, BOX_MN)
                                     : sw128_desc(sa + A_BYTES + kk * 32);
          tc_mma_f16(d_tmem, sw128_desc(sa + kk * 32), bdesc, BMN ? IDESC_BMN : IDESC,
                     (kb | kk) != 0);
        }
        issued_any = true;
        tc_commit(empty(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (failed) break;
      tc_commit(tfull(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (failed || *abort_flag) {
      *abort_flag = 1;
      if (issued_any) {  // wait until every MMA issued so far has finished
        tc_commit(drain);
        mbar_wait(drain, 0u, nullptr, 100000000ull);
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lanes 32q .. 32q+31 belong to this warp
    const int half = (warp - 2) >> 2;       // columns [128*half, 128*half + 128) of the tile
    uint8_t *const stage_epi = stage_epi_all + (warp - 2) * EPI_STAGE_BYTES;
    const int rr = lane >> 3, cc = lane & 7;
    // the hidden layer is stored with an evict-last L2 policy: GEMM2 reads it
    // back while the weights stream through L2 (measured: 2% faster)
    const uint64_t hpol = l2_evict_last_policy();
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      const int2 wt = tile_at(tile, mtotal, a.g[0].nblk, a.g[1].nblk, a.lag);
      const int which = wt.x;
      const GemmArgs &g = a.g[which];
      const int4 ti = __ldg(g.tiles + wt.y);
      const int e = ti.x, nbk = ti.w & 0xFF;
      // bias of this warp's 128 columns, lane l holding columns l, l+32, ...;
      // loaded before the wait so the latency hides behind the main loop
      float breg[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int col = nbk * BN + half * 128 + u * 32 + lane;
        breg[u] = (g.bias && col < g.N) ? __ldg(g.bias + (size_t)e * g.N + col) : 0.f;
      }
      // this warp's rows are q*32 .. q*32+31 of the tile; the row of lane l is
      // staged, the stores go out four rows at a time (rows rr, columns cc*8)
      __nv_bfloat16 *const dtile = g.D + (size_t)(ti.y + q * 32) * g.N;
      const int rows_here = ti.z - q * 32;  // valid rows of this warp (may be <= 0)
      // ReLU mask of the backward pass: this lane's row of hid, 64 columns of
      // chunk c; chunk 0's is loaded before the wait, chunk 1's while chunk 0
      // is stored
      uint32_t mk[32];
      auto load_mask = [&](int c) {
        const int col0 = nbk * BN + half * 128 + c * 64;
        const bool in = lane < rows_here && col0 < g.N;
        const uint4 *mrow = reinterpret_cast<const uint4 *>(
            g.mask + (size_t)(ti.y + q * 32 + (in ? lane : 0)) * g.N + (in ? col0 : 0));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 m4 = in && col0 + 8 * u < g.N ? __ldg(mrow + u) : make_uint4(0u, 0u, 0u, 0u);
          mk[4 * u] = m4.x; mk[4 * u + 1] = m4.y; mk[4 * u + 2] = m4.z; mk[4 * u + 3] = m4.w;
        }
      };
      if (BMN && g.mask) load_mask(0);
      // every lane waits; the outcome is made warp-uniform so that the
      // .sync.aligned tensor-memory loads below always see the full warp
      const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull(acc), acc_phase, abort_flag, kWaitNs));
      if (!ok) { failed = true; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int cl = half * 128 + c * 64;  // column inside the tile
        uint32_t v[64];
        tmem_ld64(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + cl), v);
        const int col0 = nbk * BN + cl;
        // conversion by the whole warp (the shuffles need every lane)
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float b0 = __shfl_sync(0xffffffffu, breg[2 * c + (j >> 4)], (2 * j) & 31);
          const float b1 = __shfl_sync(0xffffffffu, breg[2 * c + (j >> 4)], (2 * j + 1) & 31);
          float x0 = __uint_as_float(v[2 * j]) + b0;
          float x1 = __uint_as_float(v[2 * j + 1]) + b1;
          if (g.relu) {
            x0 = fmaxf(x0, 0.f);
            x1 = fmaxf(x1, 0.f);
          }
          if (BMN && g.mask) {  // bf16 pair: positive iff sign clear and not zero
            const uint32_t m2 = mk[j];
            if ((m2 & 0x8000u) || !(m2 & 0x7FFFu)) x0 = 0.f;
            if ((m2 & 0x80000000u) || !(m2 & 0x7FFF0000u)) x1 = 0.f;
          }
          __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
          pk[j] = *reinterpret_cast<uint32_t *>(&h);
        }
        if (BMN && g.mask && c == 0) load_mask(1);
        if (col0 < g.N && rows_here > 0) {
          // lane l's row, chunk u (8 columns) at chunk slot u ^ (l & 7)
          uint8_t *row_st = stage_epi + lane * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4 *>(row_st + ((u ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = i * 4 + rr;  // row inside the warp's block
            const uint4 v4 = *reinterpret_cast<const uint4 *>(stage_epi + r * 128 + ((cc ^ (r & 7)) << 4));
            if (r < rows_here && col0 + cc * 8 < g.N) {
              __nv_bfloat16 *dst = dtile + (size_t)r * g.N + col0 + cc * 8;
              if (!which) st_global_l2_hint(dst, v4, hpol);  // hidden layer: read back soon
              else *reinterpret_cast<uint4 *>(dst) = v4;
            }
          }
          __syncwarp();  // the block is reused by the next chunk
        }
      }
      tc_fence_before();
      mbar_arrive(tempty(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (!which) {
        // publish this warp's rows of hid to the GEMM2 tiles of the M-block:
        // the stores before the release, visible to the async proxy (TMA)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0 && (ti.w >> 8) != a.withhold_mblk) {
          atomicAdd(a.mdone + (ti.w >> 8), 1);
          atomicAdd(a.mdone + mtotal, 1);
        }
      }
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

// the wait limit of a GEMM2 tile for its M-block of hid and the test hook
// (moe_test_expert_wait); the defaults: kWaitNs, nothing withheld
std::atomic<unsigned long long> g_xwait_ns{kWaitNs};
std::atomic<int> g_withhold{-1};
unsigned long long expert_wait_limit_ns() { return g_xwait_ns.load(std::memory_order_relaxed); }
int expert_withheld_mblock() { return g_withhold.load(std::memory_order_relaxed); }

int ffn_ctas() {
  static PerDevice ctas;
  int v = 0;
  if (ctas.get([](int, int *out) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_ffn_kernel<false>,
                                                          NUM_THREADS, SMEM_BYTES) != cudaSuccess ||
            per_sm < 1)
          return MOE_ECUDA;
        *out = per_sm * num_sms();
        return MOE_OK;
      }, &v) != MOE_OK)
    return 0;
  return v;
}

}  // namespace

int launch_expert_bf16(const ExpertArgs &a, cudaStream_t st) {
  if (a.S == 0) return MOE_OK;
  static_assert(BN == kExpertBN, "tile tables assume the GEMM's N-block width");
  const int nblk1 = (a.f + BN - 1) / BN, nblk2 = (a.d + BN - 1) / BN;
  if (nblk1 > 256 || nblk2 > 256) return MOE_EINVAL;  // N-block fits the tile table's 8 bits
  if (!a.plan_ready)
    MOE_TRY(launch_expert_plan(a.offsets, a.n, const_cast<int *>(a.mprefix), a.tab1, nblk1, a.tab2,
                               nblk2, a.mdone, st));
  static PerDevice attrs;
  MOE_TRY(attrs.get([](int, int *) {
    return cudaFuncSetAttribute(expert_ffn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(expert_ffn_kernel<true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        SMEM_BYTES) == cudaSuccess
               ? MOE_OK
               : MOE_ECUDA;
  }));
  const bool bwd = a.backward != 0;
  CUtensorMap a1, b1, a2, b2;
  FfnArgs f;
  MOE_TRY(tc::make_map_2d(&a1, a.x_perm, 2, (uint64_t)a.d, (uint64_t)a.S, BM));
  MOE_TRY(tc::make_map_2d(&a2, a.hid, 2, (uint64_t)a.f, (uint64_t)a.S, BM));
  if (!bwd) {
    MOE_TRY(tc::make_map_2d(&b1, a.W1, 2, (uint64_t)a.d, (uint64_t)a.n * a.f, BN));
    MOE_TRY(tc::make_map_2d(&b2, a.W2, 2, (uint64_t)a.f, (uint64_t)a.n * a.d, BN));
    f.g[0] = GemmArgs{a.tab1, a.f, a.d, nblk1, a.b1, static_cast<__nv_bfloat16 *>(a.hid), 1, nullptr};
    f.g[1] = GemmArgs{a.tab2, a.d, a.f, nblk2, a.b2, static_cast<__nv_bfloat16 *>(a.y_perm), 0,
                      nullptr};
  } else {
    // dhid = (dy_perm W2_e) * [hid > 0]: B(n, k) = W2[e][k][n], rows e*d + k of [n*d][f];
    // dx_perm = dhid W1_e: B(n, k) = W1[e][k][n], rows e*f + k of [n*f][d]
    MOE_TRY(tc::make_map_2d(&b1, a.W2, 2, (uint64_t)a.f, (uint64_t)a.n * a.d, BK));
    MOE_TRY(tc::make_map_2d(&b2, a.W1, 2, (uint64_t)a.d, (uint64_t)a.n * a.f, BK));
    f.g[0] = GemmArgs{a.tab1, a.f, a.d, nblk1, nullptr, static_cast<__nv_bfloat16 *>(a.hid), 0,
                      static_cast<const __nv_bfloat16 *>(a.mask)};
    f.g[1] = GemmArgs{a.tab2, a.d, a.f, nblk2, nullptr, static_cast<__nv_bfloat16 *>(a.y_perm), 0,
                      nullptr};
  }
  f.mprefix = a.mprefix;
  f.n = a.n;
  f.mdone = a.mdone;
  f.status = a.status;
  f.xwait_ns = expert_wait_limit_ns();
  f.withhold_mblk = expert_withheld_mblock();
  const int64_t upper = (ceil_div(a.S, BM) + a.n) * (int64_t)(nblk1 + nblk2);
  const int ctas = ffn_ctas();
  if (ctas < 1) return MOE_ECUDA;
  const int grid = (int)(upper < ctas ? upper : ctas);
  // a GEMM2 tile follows its M-block's GEMM1 tiles by 3 or 4 waves of tiles;
  // a lag of every M-block runs all of GEMM1 first
  const int64_t mblk_upper = ceil_div(a.S, BM) + a.n;
  const int waves = (int64_t)a.S >= (int64_t)kLag4Rows * a.n ? 4 : kLagWaves;
  f.lag = (int64_t)a.S < (int64_t)kInterleaveMaxRows * a.n
              ? (int)ceil_div((int64_t)waves * grid, nblk1 + nblk2)
              : (int)(mblk_upper < INT_MAX ? mblk_upper : INT_MAX);

  // cooperative: all CTAs resident at once (a GEMM2 tile waits on other
  // CTAs' GEMM1 tiles)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int slot = -1;
  trace_begin(a.name ? a.name : (bwd ? "expert_bwd_tcgen05" : "expert_ffn_tcgen05"), st, &slot);
  const cudaError_t e = bwd ? cudaLaunchKernelEx(&cfg, expert_ffn_kernel<true>, a1, b1, a2, b2, f)
                            : cudaLaunchKernelEx(&cfg, expert_ffn_kernel<false>, a1, b1, a2, b2, f);
  trace_end(slot, st);
  count_launch();
  return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

void set_expert_wait(unsigned long long limit_ns, int withhold_mblock) {
  g_xwait_ns.store(limit_ns ? limit_ns : kWaitNs, std::memory_order_relaxed);
  g_withhold.store(withhold_mblock >= 0 ? withhold_mblock : -1, std::memory_order_relaxed);
}

}  // namespace moe
