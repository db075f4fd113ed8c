// dispatch.cu -- sending every (token, slot) pair to its expert.
//
// [SGMoE-note] "Sparsely-Gated MoE 层架构": E_i(x) is not evaluated where
// G(x)_i = 0, so only the kept (token, expert) pairs are routed.  [MoE-deep]
// §3.2: an expert takes at most C pairs; the rest overflow.
//
// Pairs are visited in (token, slot) order.  The r-th pair of expert e goes to
// row offsets[e] + r when r < C, offsets being the exclusive scan of
// min(count, C): a stable counting sort, built from
//   1. dispatch_hist      per-block histograms hist[b][e] (shared-memory atomics;
//                         counts are order-free)
//   2. dispatch_scan_cols base[b][e] = sum of hist[b'][e] over b' < b (one thread
//                         per expert, blocks in order), counts[e]
//   3. dispatch_offsets   one block: offsets / uncapped offsets / tile prefixes
//   4. dispatch_rank      per block, one warp walks the block's pairs in order
//                         (32 at a time, __match_any_sync groups equal experts)
//                         and assigns ranks -> row_of, perm_token, sorted gates
//   5. dispatch_gather    x rows copied (and cast) into their rows, one warp
//                         per token, 16-byte stores
// No step depends on scheduling order, so the permutation is deterministic.
#include <limits.h>

#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

__global__ void dispatch_hist_kernel(const int *idx, int T, int k, int n, int tpb, int *hist,
                                     int *status) {
  extern __shared__ int sh[];
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < n; e += NT) sh[e] = 0;
  __syncthreads();
  const int64_t p0 = (int64_t)b * tpb * k;
  const int64_t p1 = min((int64_t)(b + 1) * tpb, (int64_t)T) * k;
  bool bad = false;
  for (int64_t p = p0 + threadIdx.x; p < p1; p += NT) {
    const int e = idx[p];
    if (e >= 0 && e < n) atomicAdd(&sh[e], 1);
    else bad = true;
  }
  if (bad && status) atomicOr(status, MOE_STATUS_BAD_INDEX);
  __syncthreads();
  int *out = hist + (size_t)b * n;
  for (int e = threadIdx.x; e < n; e += NT) out[e] = sh[e];
}

// base[b][e] = sum of hist[b'][e] over b' < b.  A block takes 32 experts
// (coalesced columns) and splits the B blocks into SC contiguous ranges:
// range sums, their prefix in shared memory, then a second pass writes the
// bases.  counts[e] = the total.
constexpr int SC = 32;
__global__ void __launch_bounds__(32 * SC) dispatch_scan_cols_kernel(const int *hist, int B, int n,
                                                                     int *base, int *counts) {
  __shared__ int tot[SC][33];
  const int e = blockIdx.x * 32 + threadIdx.x;
  const int r = threadIdx.y;
  const int chunk = (B + SC - 1) / SC;
  const int b0 = min(B, r * chunk), b1 = min(B, b0 + chunk);
  int s = 0;
  if (e < n)
    for (int b = b0; b < b1; ++b) s += hist[(size_t)b * n + e];
  tot[r][threadIdx.x] = s;
  __syncthreads();
  int run = 0;
  for (int q = 0; q < r; ++q) run += tot[q][threadIdx.x];
  if (e >= n) return;
  for (int b = b0; b < b1; ++b) {
    const int h = hist[(size_t)b * n + e];
    base[(size_t)b * n + e] = run;
    run += h;
  }
  if (r == SC - 1) counts[e] = run;
}

// Block-wide exclusive scan: returns the sum of `v` over all threads with a
// lower index.  Every thread of the block must call it.
__device__ __forceinline__ long long block_exclusive_scan(long long v) {
  __shared__ long long warp_tot[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nwarps = (int)(blockDim.x >> 5);
  long long inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    const long long t = lane < nwarps ? warp_tot[lane] : 0;
    long long ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    warp_tot[lane] = ti - t;
  }
  __syncthreads();
  const long long res = warp_tot[w] + inc - v;
  __syncthreads();  // warp_tot is reused by the next call
  return res;
}

constexpr int SCAN_NT = 1024, SCAN_PER = 8;  // n <= 8192

// offsets[e] = sum_{e'<e} min(count, C); ucoff: the same without the cap;
// seg_mblk / seg_tiles: exclusive scans of ceil(kept/rows).
// One expert's tiles of a grouped GEMM: N-block major, M-block minor.
__device__ __forceinline__ void write_tiles(int4 *tab, int nblk, int e, int mb_base, int mbe,
                                            int row_base, int rows) {
  for (int nbk = 0; nbk < nblk; ++nbk)
    for (int mb = 0; mb < mbe; ++mb)
      tab[(size_t)(mb_base * nblk + nbk * mbe + mb)] =
          make_int4(e, row_base + mb * kExpertBM, min(kExpertBM, rows - mb * kExpertBM), nbk);
}

__global__ void __launch_bounds__(SCAN_NT) dispatch_offsets_kernel(
    const int *counts, int n, long long C, int *offsets, int *ucoff, int *seg_mblk, int mblk_rows,
    int *seg_tiles, int tile_rows, int4 *tab1, int nblk1, int4 *tab2, int nblk2) {
  // each thread takes a contiguous run of per <= SCAN_PER experts, so that
  // small n still spreads over the whole block
  const int per = (n + SCAN_NT - 1) / SCAN_NT;
  const int e0 = threadIdx.x * per;
  auto values = [&](int e, long long &raw, long long &kept, long long &mb, long long &tl) {
    raw = e < n ? counts[e] : 0;
    kept = raw < C ? raw : C;
    mb = mblk_rows > 0 ? (kept + mblk_rows - 1) / mblk_rows : 0;
    tl = tile_rows > 0 ? (kept + tile_rows - 1) / tile_rows : 0;
  };
  long long sk = 0, sr = 0, sm = 0, st = 0;
  for (int j = 0; j < per; ++j) {
    long long raw, kept, mb, tl;
    values(e0 + j, raw, kept, mb, tl);
    sk += kept; sr += raw; sm += mb; st += tl;
  }
  long long p = block_exclusive_scan(sk);
  long long q = block_exclusive_scan(sr);
  long long pm = block_exclusive_scan(sm);
  long long pt = block_exclusive_scan(st);
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    long long raw, kept, mb, tl;
    values(e, raw, kept, mb, tl);
    if (e < n) {
      offsets[e] = (int)p;
      ucoff[e] = (int)q;
      if (seg_mblk) seg_mblk[e] = (int)pm;
      if (seg_tiles) seg_tiles[e] = (int)pt;
      if (tab1) {  // expert GEMM tile tables
        write_tiles(tab1, nblk1, e, (int)pm, (int)mb, (int)p, (int)kept);
        write_tiles(tab2, nblk2, e, (int)pm, (int)mb, (int)p, (int)kept);
      }
    }
    p += kept;
    q += raw;
    pm += mb;
    pt += tl;
    if (e == n - 1) {
      offsets[n] = (int)p;
      ucoff[n] = (int)q;
      if (seg_mblk) seg_mblk[n] = (int)pm;
      if (seg_tiles) seg_tiles[n] = (int)pt;
    }
  }
}

__global__ void dispatch_rank_kernel(const int *idx, const float *gate, int T, int k, int n,
                                     int tpb, long long C, const int *base, const int *offsets,
                                     const int *ucoff, int *row_of, int *perm_token,
                                     int *perm_slot, float *gate_sorted) {
  extern __shared__ int cnt[];  // [n] ranks handed out so far in this block
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < n; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int64_t p0 = (int64_t)b * tpb * k;
  const int64_t p1 = min((int64_t)(b + 1) * tpb, (int64_t)T) * k;
  const int *bbase = base + (size_t)b * n;
  for (int64_t q = p0; q < p1; q += 32) {
    const int64_t p = q + lane;
    const bool valid = p < p1;
    const int e = valid ? idx[p] : -1;
    const bool ok = valid && e >= 0 && e < n;
    const unsigned grp = __match_any_sync(0xffffffffu, ok ? e : n + lane);
    const int before_me = __popc(grp & lt_mask);
    const int r_local = ok ? cnt[e] + before_me : 0;
    __syncwarp();
    if (ok && before_me == 0) cnt[e] += __popc(grp);
    __syncwarp();
    if (!valid) continue;
    if (!ok) {
      row_of[p] = -1;
      continue;
    }
    const int rank = bbase[e] + r_local;
    if (gate_sorted) gate_sorted[ucoff[e] + rank] = gate[p];
    if ((long long)rank < C) {
      const int row = offsets[e] + rank;
      row_of[p] = row;
      perm_token[row] = (int)(p / k);
      if (perm_slot) perm_slot[row] = (int)(p % k);
    } else {
      row_of[p] = -1;
    }
  }
}

// x rows into their expert rows, cast to the expert dtype; warp per token.
template <bool BF16>
__global__ void dispatch_gather_kernel(const float *x, const int *row_of, int T, int k, int d,
                                       void *x_perm) {
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int rows[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) rows[j] = j < k ? row_of[(size_t)t * k + j] : -1;
  const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)t * d);
  const int nchunk = d >> 3;  // 8 elements per chunk
  for (int c = lane; c < nchunk; c += 32) {
    const float4 u = __ldg(xr + 2 * c), v = __ldg(xr + 2 * c + 1);
    if (BF16) {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(u.x, u.y), p1 = __floats2bfloat162_rn(u.z, u.w);
      __nv_bfloat162 p2 = __floats2bfloat162_rn(v.x, v.y), p3 = __floats2bfloat162_rn(v.z, v.w);
      uint4 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&p0);
      pk.y = *reinterpret_cast<uint32_t *>(&p1);
      pk.z = *reinterpret_cast<uint32_t *>(&p2);
      pk.w = *reinterpret_cast<uint32_t *>(&p3);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (rows[j] >= 0)
          reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(x_perm) + (size_t)rows[j] * d)[c] = pk;
    } else {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (rows[j] >= 0) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(x_perm) + (size_t)rows[j] * d);
          dst[2 * c] = u;
          dst[2 * c + 1] = v;
        }
    }
  }
}

__global__ void __launch_bounds__(SCAN_NT) expert_plan_kernel(const int *offsets, int n,
                                                              int *mprefix, int4 *tab1, int nblk1,
                                                              int4 *tab2, int nblk2) {
  const int per = (n + SCAN_NT - 1) / SCAN_NT;
  const int e0 = threadIdx.x * per;
  auto rows = [&](int e) -> long long { return e < n ? (long long)(offsets[e + 1] - offsets[e]) : 0; };
  long long sm = 0;
  for (int j = 0; j < per; ++j) sm += (rows(e0 + j) + kExpertBM - 1) / kExpertBM;
  long long p = block_exclusive_scan(sm);
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    const long long m = rows(e), mb = (m + kExpertBM - 1) / kExpertBM;
    if (e < n) {
      mprefix[e] = (int)p;
      write_tiles(tab1, nblk1, e, (int)p, (int)mb, offsets[e], (int)m);
      write_tiles(tab2, nblk2, e, (int)p, (int)mb, offsets[e], (int)m);
    }
    p += mb;
    if (e == n - 1) mprefix[n] = (int)p;
  }
}

}  // namespace

int dispatch_tokens_per_block(int T) {
  // about two blocks per SM of a 148-SM part, 32..256 tokens each
  int64_t tpb = ceil_div(ceil_div(T, 296), 32) * 32;
  if (tpb < 32) tpb = 32;
  if (tpb > 256) tpb = 256;
  return (int)tpb;
}

int launch_dispatch(const DispatchArgs &a, cudaStream_t st) {
  if (a.n > SCAN_NT * SCAN_PER) return MOE_EINVAL;
  const int tpb = dispatch_tokens_per_block(a.T);
  const int B = (int)ceil_div(a.T, tpb);
  const size_t sh = sizeof(int) * a.n;
  if (B > 0) {
    MOE_TRY(launch("dispatch_hist", dispatch_hist_kernel, dim3(B), dim3(NT), sh, st, a.idx, a.T,
                   a.k, a.n, tpb, a.hist, a.status));
    MOE_TRY(launch("dispatch_scan_cols", dispatch_scan_cols_kernel,
                   dim3((unsigned)ceil_div(a.n, 32)), dim3(32, SC), 0, st, (const int *)a.hist, B,
                   a.n, a.base, a.counts));
  } else {
    cudaMemsetAsync(a.counts, 0, sizeof(int) * a.n, st);
  }
  const long long C = a.C;
  MOE_TRY(launch("dispatch_offsets", dispatch_offsets_kernel, dim3(1), dim3(SCAN_NT), 0, st,
                 (const int *)a.counts, a.n, C, a.offsets, a.ucoff, a.seg_mblk, a.mblk_rows,
                 a.seg_tiles, a.tile_rows, a.tab1, a.nblk1, a.tab2, a.nblk2));
  if (B > 0)
    MOE_TRY(launch("dispatch_rank", dispatch_rank_kernel, dim3(B), dim3(128), sh, st, a.idx,
                   a.gate, a.T, a.k, a.n, tpb, C, (const int *)a.base, (const int *)a.offsets,
                   (const int *)a.ucoff, a.row_of, a.perm_token, a.perm_slot, a.gate_sorted));
  return MOE_OK;
}

int launch_gather(const float *x, const int *row_of, int T, int k, int d, int bf16, void *x_perm,
                  cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(T, NT / 32));
  if (bf16)
    return launch("dispatch_gather", dispatch_gather_kernel<true>, grid, dim3(NT), 0, st, x,
                  row_of, T, k, d, x_perm);
  return launch("dispatch_gather", dispatch_gather_kernel<false>, grid, dim3(NT), 0, st, x, row_of,
                T, k, d, x_perm);
}

int launch_expert_plan(const int *offsets, int n, int *mprefix, int4 *tab1, int nblk1, int4 *tab2,
                       int nblk2, cudaStream_t st) {
  if (n > SCAN_NT * SCAN_PER) return MOE_EINVAL;
  return launch("expert_plan", expert_plan_kernel, dim3(1), dim3(SCAN_NT), 0, st, offsets, n,
                mprefix, tab1, nblk1, tab2, nblk2);
}

}  // namespace moe
