// dispatch.cu -- sending every (token, slot) pair to its expert.
//
// [SGMoE-note] "Sparsely-Gated MoE 层架构": E_i(x) is not evaluated where
// G(x)_i = 0, so only the kept (token, expert) pairs are routed.  [MoE-deep]
// §3.2: an expert takes at most C pairs; the rest overflow.
//
// Pairs are visited in (token, slot) order.  The r-th pair of expert e goes to
// row offsets[e] + r when r < C, offsets being the exclusive scan of
// min(count, C): a stable counting sort over blocks of tpb tokens, in three
// launches:
//   1. dispatch_hist   per block: the block's expert ids staged in shared
//                      memory, one warp walks its pairs in order (32 at a time,
//                      __match_any_sync groups equal experts) and hands out
//                      the rank of every pair among the block's pairs of the
//                      same expert (kept in row_of until step 3) -> hist[b][e]
//   2. dispatch_scan   base[b][e] = sum of hist[b'][e] over b' < b, counts[e];
//                      the last block to finish (atomic ticket, no waiting)
//                      then writes offsets / uncapped offsets / tile prefixes
//                      and the expert GEMM tile tables
//   3. dispatch_place  one warp per token: rank = base[b][e] + block rank ->
//                      row_of, perm_token, sorted gates; optionally the token's
//                      x row copied (and cast) into its expert rows, and into
//                      row t of the shared expert's input, 16-byte stores
// No step depends on scheduling order, so the permutation is deterministic.
#include <limits.h>

#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

// smem: cnt[n] then the block's ids [tpb * k]
__global__ void __launch_bounds__(NT) dispatch_hist_kernel(const int *idx, int T, int k, int n,
                                                           int tpb, int *hist, int *brank,
                                                           int *ticket, int *status) {
  extern __shared__ int sh[];
  int *cnt = sh, *ids = sh + n;
  const int b = blockIdx.x;
  if (b == 0 && threadIdx.x == 0) *ticket = 0;  // the scan kernel's last-block election
  const int64_t p0 = (int64_t)b * tpb * k;
  const int np = (int)(min((int64_t)(b + 1) * tpb, (int64_t)T) * k - p0);
  for (int e = threadIdx.x; e < n; e += NT) cnt[e] = 0;
  for (int i = threadIdx.x; i < np; i += NT) ids[i] = idx[p0 + i];
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const unsigned lt_mask = (1u << lane) - 1u;
    bool bad = false;
    for (int q = 0; q < np; q += 32) {
      const int i = q + lane;
      const bool valid = i < np;
      const int e = valid ? ids[i] : -1;
      const bool ok = valid && e >= 0 && e < n;
      const unsigned grp = __match_any_sync(0xffffffffu, ok ? e : n + lane);
      const int before_me = __popc(grp & lt_mask);
      const int r_local = ok ? cnt[e] + before_me : -1;  // -1: an id outside [0, n)
      __syncwarp();
      if (ok && before_me == 0) cnt[e] += __popc(grp);
      __syncwarp();
      if (valid) brank[p0 + i] = r_local;
      bad |= valid && !ok;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_INDEX);
  }
  __syncthreads();
  int *out = hist + (size_t)b * n;
  for (int e = threadIdx.x; e < n; e += NT) out[e] = cnt[e];
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

// Four block-wide exclusive scans at once (one set of barriers): v[i] is
// replaced by the sum of v[i] over all threads with a lower index.
__device__ __forceinline__ void block_exclusive_scan4(long long (&v)[4]) {
  __shared__ long long warp_tot[4][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nwarps = (int)(blockDim.x >> 5);
  long long inc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    inc[i] = v[i];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, inc[i], off);
      if (lane >= off) inc[i] += o;
    }
    if (lane == 31) warp_tot[i][w] = inc[i];
  }
  __syncthreads();
  if (w < 4) {  // warp i scans the warp totals of value i
    const long long t = lane < nwarps ? warp_tot[w][lane] : 0;
    long long ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    warp_tot[w][lane] = ti - t;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = warp_tot[i][w] + inc[i] - v[i];
  __syncthreads();  // warp_tot is reused by the next call
}

constexpr int SCAN_NT = 1024, SCAN_PER = 8;  // n <= 8192

// One expert's tiles of a grouped GEMM: entry (global M-block) * nblk + N-block;
// the last field packs the N-block (8 bits) and the global M-block index.
__device__ __forceinline__ void write_tiles(int4 *tab, int nblk, int e, int mb_base, int mbe,
                                            int row_base, int rows) {
  for (int mb = 0; mb < mbe; ++mb)
    for (int nbk = 0; nbk < nblk; ++nbk)
      tab[(size_t)(mb_base + mb) * nblk + nbk] =
          make_int4(e, row_base + mb * kExpertBM, min(kExpertBM, rows - mb * kExpertBM),
                    nbk | ((mb_base + mb) << 8));
}

struct PlanOut {
  long long C;
  int *offsets, *ucoff, *seg_mblk, *seg_tiles;
  int mblk_rows, tile_rows;
  int4 *tab1, *tab2;
  int nblk1, nblk2;
  int *mdone;  // with the tables: per-M-block counters of the expert GEMM, zeroed
};

// offsets[e] = sum_{e'<e} min(count, C); ucoff: the same without the cap;
// seg_mblk / seg_tiles: exclusive scans of ceil(kept/rows); the expert GEMM
// tile tables.  Run by one whole block of SCAN_NT threads.
__device__ void write_plan(const int *counts, int n, const PlanOut &o) {
  const long long C = o.C;
  int *offsets = o.offsets, *ucoff = o.ucoff, *seg_mblk = o.seg_mblk, *seg_tiles = o.seg_tiles;
  const int mblk_rows = o.mblk_rows, tile_rows = o.tile_rows;
  int4 *tab1 = o.tab1, *tab2 = o.tab2;
  const int nblk1 = o.nblk1, nblk2 = o.nblk2;
  int *mdone = o.mdone;
  // each thread takes a contiguous run of per <= SCAN_PER experts, so that
  // small n still spreads over the whole block
  const int per = (n + SCAN_NT - 1) / SCAN_NT;
  const int e0 = threadIdx.x * per;
  auto values = [&](int e, long long &raw, long long &kept, long long &mb, long long &tl) {
    raw = e < n ? __ldcg(counts + e) : 0;
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
  long long sc[4] = {sk, sr, sm, st};
  block_exclusive_scan4(sc);
  long long p = sc[0], q = sc[1], pm = sc[2], pt = sc[3];
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    long long raw, kept, mb, tl;
    values(e, raw, kept, mb, tl);
    if (e < n) {
      offsets[e] = (int)p;
      ucoff[e] = (int)q;
      if (seg_mblk) seg_mblk[e] = (int)pm;
      if (seg_tiles) seg_tiles[e] = (int)pt;
      if (tab1 && !(seg_mblk && mblk_rows == kExpertBM)) {  // else dispatch_tiles_kernel
        write_tiles(tab1, nblk1, e, (int)pm, (int)mb, (int)p, (int)kept);
        write_tiles(tab2, nblk2, e, (int)pm, (int)mb, (int)p, (int)kept);
        for (long long j = 0; j < mb; ++j) mdone[pm + j] = 0;
        if (e == n - 1) mdone[pm + mb] = 0;  // the count over all M-blocks
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

// base[b][e] = sum of hist[b'][e] over b' < b.  A block takes 32 experts
// (coalesced columns) and splits the B blocks into SC contiguous ranges:
// range sums, their prefix in shared memory, then a second pass writes the
// bases.  counts[e] = the total.  The last block to finish writes the plan.
constexpr int SC = SCAN_NT / 32;
__global__ void __launch_bounds__(SCAN_NT) dispatch_scan_kernel(const int *hist, int B, int n,
                                                                int *base, int *counts,
                                                                int *ticket, PlanOut o) {
  __shared__ int tot[SC][33];
  __shared__ int last;
  const int tx = threadIdx.x & 31, r = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + tx;
  const int chunk = (B + SC - 1) / SC;
  const int b0 = min(B, r * chunk), b1 = min(B, b0 + chunk);
  // the range is read in batches of 8 independent loads (the sums are exact
  // integer sums, so batching changes nothing)
  constexpr int VB = 8;
  int s = 0;
  if (e < n)
    for (int b = b0; b < b1; b += VB) {
      int h[VB];
#pragma unroll
      for (int j = 0; j < VB; ++j) h[j] = b + j < b1 ? hist[(size_t)(b + j) * n + e] : 0;
#pragma unroll
      for (int j = 0; j < VB; ++j) s += h[j];
    }
  tot[r][tx] = s;
  __syncthreads();
  int run = 0;
  for (int q = 0; q < r; ++q) run += tot[q][tx];
  if (e < n) {
    for (int b = b0; b < b1; b += VB) {
      int h[VB];
#pragma unroll
      for (int j = 0; j < VB; ++j) h[j] = b + j < b1 ? hist[(size_t)(b + j) * n + e] : 0;
#pragma unroll
      for (int j = 0; j < VB; ++j) {
        if (b + j < b1) base[(size_t)(b + j) * n + e] = run;
        run += h[j];
      }
    }
    if (r == SC - 1) counts[e] = run;
  }
  // counts visible device-wide before the ticket is taken
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  write_plan(counts, n, o);
}

// One warp per token.  Lanes j < k finish the pairs of the token (row_of
// holds each pair's rank inside its block on entry, its row on exit); with
// COPY the whole warp then writes the token's x row into its expert rows,
// cast to bf16 for the tensor-core experts.
template <bool COPY, bool BF16>
__global__ void __launch_bounds__(NT) dispatch_place_kernel(
    const int *idx, const float *gate, int T, int k, int n, int tpb, long long C,
    const int *base, const int *offsets, const int *ucoff, int *row_of, int *perm_token,
    int *perm_slot, float *gate_sorted, const float *x, int d, void *x_perm, void *x_shared,
    int *shared_off, int *shared_mprefix, int4 *shared_tab1, int4 *shared_tab2, int *shared_mdone,
    int nblk1, int nblk2) {
  if (shared_off && blockIdx.x == 0) {
    // the shared expert: rows 0..T-1 in token order, its tile tables and
    // counters (one expert, mbe M-blocks; see write_tiles)
    const int mbe = (T + kExpertBM - 1) / kExpertBM;
    if (threadIdx.x == 0) {
      shared_off[0] = 0;
      shared_off[1] = T;
      shared_mprefix[0] = 0;
      shared_mprefix[1] = mbe;
    }
    for (int i = threadIdx.x; i < mbe * nblk1; i += NT) {
      const int mb = i / nblk1, nbk = i - mb * nblk1;  // entry: M-block * nblk + N-block
      shared_tab1[i] = make_int4(0, mb * kExpertBM, min(kExpertBM, T - mb * kExpertBM), nbk | (mb << 8));
    }
    for (int i = threadIdx.x; i < mbe * nblk2; i += NT) {
      const int mb = i / nblk2, nbk = i - mb * nblk2;
      shared_tab2[i] = make_int4(0, mb * kExpertBM, min(kExpertBM, T - mb * kExpertBM), nbk | (mb << 8));
    }
    for (int i = threadIdx.x; i <= mbe; i += NT) shared_mdone[i] = 0;
  }
  const int t = blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  // the token's first x chunk is requested before the rank lookups below
  const float4 *xr = COPY ? reinterpret_cast<const float4 *>(x + (size_t)t * d) : nullptr;
  const int nchunk = d >> 3;  // 8 elements per chunk
  float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), v0 = u0;
  if (COPY && lane < nchunk) {
    u0 = __ldg(xr + 2 * lane);
    v0 = __ldg(xr + 2 * lane + 1);
  }
  int myrow = -1;
  if (lane < k) {
    const int64_t p = (int64_t)t * k + lane;
    const int r_local = row_of[p];
    if (r_local >= 0) {
      const int e = idx[p];
      const int rank = base[(size_t)(t / tpb) * n + e] + r_local;
      if (gate_sorted) gate_sorted[ucoff[e] + rank] = gate[p];
      if ((long long)rank < C) {
        myrow = offsets[e] + rank;
        perm_token[myrow] = t;
        if (perm_slot) perm_slot[myrow] = lane;
      }
    }
    row_of[p] = myrow;
  }
  if constexpr (COPY) {
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const int v = __shfl_sync(0xffffffffu, myrow, j);
      rows[j] = j < k ? v : -1;
    }
    for (int c = lane; c < nchunk; c += 32) {
      const float4 u = c == lane ? u0 : __ldg(xr + 2 * c);
      const float4 v = c == lane ? v0 : __ldg(xr + 2 * c + 1);
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
        if (x_shared)
          reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(x_shared) + (size_t)t * d)[c] = pk;
      } else {
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
          if (rows[j] >= 0) {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(x_perm) + (size_t)rows[j] * d);
            dst[2 * c] = u;
            dst[2 * c + 1] = v;
          }
        if (x_shared) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(x_shared) + (size_t)t * d);
          dst[2 * c] = u;
          dst[2 * c + 1] = v;
        }
      }
    }
  }
}

// The expert GEMM's tile tables from the offsets and M-block prefix the scan
// wrote: one thread per expert, so the tables (six 16-byte entries an expert
// at d = 512, f = 1024) are written by many SMs instead of the scan's last block.
__global__ void dispatch_tiles_kernel(const int *offsets, const int *mprefix, int n, int4 *tab1,
                                      int nblk1, int4 *tab2, int nblk2, int *mdone) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int row = offsets[e], rows = offsets[e + 1] - row;
  const int mb_base = mprefix[e], mb = mprefix[e + 1] - mb_base;
  write_tiles(tab1, nblk1, e, mb_base, mb, row, rows);
  write_tiles(tab2, nblk2, e, mb_base, mb, row, rows);
  for (int j = 0; j < mb; ++j) mdone[mb_base + j] = 0;
  if (e == n - 1) mdone[mb_base + mb] = 0;  // the count over all M-blocks
}

__global__ void __launch_bounds__(SCAN_NT) expert_plan_kernel(const int *offsets, int n,
                                                              int *mprefix, int4 *tab1, int nblk1,
                                                              int4 *tab2, int nblk2, int *mdone) {
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
      for (long long j = 0; j < mb; ++j) mdone[p + j] = 0;
      if (e == n - 1) mdone[p + mb] = 0;  // the count over all M-blocks
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
  if (a.T > 0 && a.x && (!a.x_perm || a.d % 8)) return MOE_EINVAL;
  const int tpb = dispatch_tokens_per_block(a.T);
  const int B = (int)ceil_div(a.T, tpb);
  if (B > 0) {
    const size_t sh = sizeof(int) * ((size_t)a.n + (size_t)tpb * a.k);
    MOE_TRY(launch("dispatch_hist", dispatch_hist_kernel, dim3(B), dim3(NT), sh, st, a.idx, a.T,
                   a.k, a.n, tpb, a.hist, a.row_of, a.ticket, a.status));
  } else if (cudaMemsetAsync(a.ticket, 0, sizeof(int), st) != cudaSuccess) {
    return MOE_ECUDA;
  }
  PlanOut o;
  o.C = a.C;
  o.offsets = a.offsets;
  o.ucoff = a.ucoff;
  o.seg_mblk = a.seg_mblk;
  o.seg_tiles = a.seg_tiles;
  o.mblk_rows = a.mblk_rows;
  o.tile_rows = a.tile_rows;
  o.tab1 = a.tab1;
  o.tab2 = a.tab2;
  o.nblk1 = a.nblk1;
  o.nblk2 = a.nblk2;
  o.mdone = a.mdone;
  MOE_TRY(launch("dispatch_scan", dispatch_scan_kernel, dim3((unsigned)ceil_div(a.n, 32)),
                 dim3(SCAN_NT), 0, st, (const int *)a.hist, B, a.n, a.base, a.counts, a.ticket, o));
  if (a.tab1 && a.seg_mblk && a.mblk_rows == kExpertBM)  // the tile tables, off the scan's last block
    MOE_TRY(launch("dispatch_tiles", dispatch_tiles_kernel, dim3((unsigned)ceil_div(a.n, 128)),
                   dim3(128), 0, st, (const int *)a.offsets, (const int *)a.seg_mblk, a.n, a.tab1,
                   a.nblk1, a.tab2, a.nblk2, a.mdone));
  if (B == 0) return MOE_OK;
  const dim3 grid((unsigned)ceil_div(a.T, NT / 32));
  const long long C = a.C;
  auto place = [&](auto kern) {
    return launch("dispatch_place", kern, grid, dim3(NT), 0, st, a.idx, a.gate, a.T, a.k, a.n, tpb,
                  C, (const int *)a.base, (const int *)a.offsets, (const int *)a.ucoff, a.row_of,
                  a.perm_token, a.perm_slot, a.gate_sorted, a.x, a.d, a.x_perm, a.x_shared,
                  a.shared_off, a.shared_mprefix, a.shared_tab1, a.shared_tab2, a.shared_mdone,
                  a.nblk1, a.nblk2);
  };
  if (!a.x) return place(dispatch_place_kernel<false, false>);
  if (a.x_bf16) return place(dispatch_place_kernel<true, true>);
  return place(dispatch_place_kernel<true, false>);
}

int launch_expert_plan(const int *offsets, int n, int *mprefix, int4 *tab1, int nblk1, int4 *tab2,
                       int nblk2, int *mdone, cudaStream_t st) {
  if (n > SCAN_NT * SCAN_PER) return MOE_EINVAL;
  return launch("expert_plan", expert_plan_kernel, dim3(1), dim3(SCAN_NT), 0, st, offsets, n,
                mprefix, tab1, nblk1, tab2, nblk2, mdone);
}

}  // namespace moe
