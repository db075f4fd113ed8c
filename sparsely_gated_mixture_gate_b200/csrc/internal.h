// internal.h -- declarations shared by the library's translation units.
// Not part of the ABI (that is include/moe.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- launches
// Every kernel goes through launch(): it counts the launch, records CUDA
// events around it when tracing is on, and turns a launch error into
// MOE_ECUDA.
void trace_begin(const char *name, cudaStream_t st, int *slot);
void trace_end(int slot, cudaStream_t st);
void count_launch();

template <class Kernel, class... Args>
int launch(const char *name, Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
           Args... args) {
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return MOE_OK;
  int slot = -1;
  trace_begin(name, st, &slot);
  kernel<<<grid, block, smem, st>>>(args...);
  cudaError_t e = cudaGetLastError();
  trace_end(slot, st);
  count_launch();
  return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

#define MOE_TRY(expr)            \
  do {                           \
    int _rc = (expr);            \
    if (_rc != MOE_OK) return _rc; \
  } while (0)

// A value worked out once per device (a kernel attribute set, an occupancy,
// a device check) and shared by every host thread: get() runs make(dev, &v)
// for the current device the first time, under a lock, and returns the
// stored value afterwards.  A failed make() stores nothing.
constexpr int kMaxDevices = 64;
class PerDevice {
 public:
  template <class F>
  int get(F make, int *out = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_EDEVICE;
    std::lock_guard<std::mutex> lock(mu_);
    if (!done_[dev]) {
      int v = 0;
      const int rc = make(dev, &v);
      if (rc != MOE_OK) return rc;
      val_[dev] = v;
      done_[dev] = true;
    }
    if (out) *out = val_[dev];
    return MOE_OK;
  }

 private:
  std::mutex mu_;
  bool done_[kMaxDevices] = {};
  int val_[kMaxDevices] = {};
};

// MOE_OK when the current device is an sm_100 part (the library's only
// target), else MOE_EDEVICE; checked once per device.
int check_device();

int num_sms();

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- tiling constants
constexpr int kGateBM = 128, kGateBN = 128;   // SIMT gate GEMM tile
constexpr int kExpertBM = 128;                // tcgen05 grouped GEMM rows per tile
constexpr int kMaxK = 8;                      // largest supported top-k

// tokens per dispatch block, rows per routing tile: functions of the sizes
// only, so results never depend on the device.
int dispatch_tokens_per_block(int T);
int route_rows_per_tile(int R);

// ---------------------------------------------------------------- kernels (host launchers)
struct GateGemmArgs {
  const float *x;          // [T][d]
  int d;
  const int *row_token;    // [R] token of every GEMM row, or nullptr (row r = token r)
  const int *seg_off;      // [G+1] first row of every group, or nullptr (one group of R rows)
  const int *seg_mblk;     // [G+1] exclusive scan of ceil(rows_g / kGateBM), or nullptr
  int R, G;
  const float *Wg, *Wn, *bias;  // group g: Wg + g*d*nb, Wn + g*d*nb, bias + g*nb
  int nb, noise;
  float *c, *s;            // [R][nb]
  int *status;
};
int launch_gate_gemm(const GateGemmArgs &a, int mblk_upper, cudaStream_t st);
// the same on the tensor cores (three-pass TF32 split); xhi/xlo: [R][d],
// whi/wlo: [G][nb*(noise?2:1)][d] scratch
int launch_gate_tf32x3(const GateGemmArgs &a, int mblk_upper, float *xhi, float *xlo, float *whi,
                       float *wlo, cudaStream_t st);

struct RouteArgs {
  const float *c, *s;      // [R][nb]
  int R, nb, k, router, noise;
  uint64_t seed;
  const unsigned long long *seed_dev;  // when set, the noise key is read here at run time
  uint32_t token_base;     // added to the token index in the noise counter
  const int *row_token;    // [R] or nullptr
  const int *row_slot;     // [R] primary slot of the row (secondary gate), or nullptr
  const int *seg_off;      // [G+1] or nullptr
  const int *seg_tiles;    // [G+1] exclusive scan of ceil(rows_g / RT), or nullptr
  int G, RT;
  int secondary;           // 0: gate id 0; 1: gate id 1 + group
  int *out_idx;            // [T][K]
  float *out_gate;         // [T][K]
  int K;                   // slots per token in out_idx/out_gate
  int expert_stride;       // secondary: expert id = g * expert_stride + j
  const float *gate_mult;  // secondary: primary gates [T][k1]
  int k1;
  float *load_part;        // [tiles][nb]
  float *psum_part;        // [tiles][nb] or nullptr
  const float *sel_bias;   // sigmoid router: [nb] selection bias, or nullptr
  float *stats_part;       // [tiles][2] or nullptr: per tile, sum over rows of |c|^2
                           // and of the entropy of softmax(c)
  int4 *kth;               // [R] or nullptr: per row {H of the (k+1)-th ranked, its id,
                           // H of the k-th, its id} (H bits as int; -inf / INT_MAX if absent)
  float *gate_raw;         // [R][k] or nullptr: the row's own gates (the secondary gate's,
  int *idx_raw;            // before the primary factor) and kept ids, by row (backward)
  int *status;
};
int launch_route(const RouteArgs &a, int tiles_upper, cudaStream_t st);
// out[g][j] = sum over the tiles of group g (in order) of part[tile][j]
int launch_route_reduce(const float *part, const int *seg_tiles, int G, int ntiles_flat, int nb,
                        float *out, cudaStream_t st);
// Hierarchical load: load[g*b+j] = cnt_g ? load_p[g] * load2[g*b+j] / cnt_g : 0
int launch_hier_load(const float *load_p, const float *load2, const int *cnt, int a, int b,
                     float *load, cudaStream_t st);

struct DispatchArgs {
  const int *idx;          // [T][k]
  int T, k, n;
  int64_t C;               // capacity (INT64_MAX: none)
  const float *gate;       // [T][k] or nullptr; with it gate_sorted is written
  int *hist, *base;        // [B][n] scratch
  int *counts;             // [n]
  int *offsets;            // [n+1]
  int *ucoff;              // [n+1] scratch (uncapped offsets)
  int *perm_token;         // [T*k]
  int *perm_slot;          // [T*k] or nullptr
  int *row_of;             // [T][k]
  float *gate_sorted;      // [T*k] or nullptr
  int *seg_mblk;           // [n+1] or nullptr: exclusive scan of ceil(kept_e / mblk_rows)
  int mblk_rows;
  int *seg_tiles;          // [n+1] or nullptr: exclusive scan of ceil(kept_e / tile_rows)
  int tile_rows;
  int4 *tab1, *tab2;       // expert GEMM tile tables (see ExpertArgs), or nullptr
  int nblk1, nblk2;
  int *mdone;              // with the tables: per-M-block counters, zeroed
  int *ticket;             // one int of scratch (last-block election of the scan)
  const float *x;          // [T][d] or nullptr: with it x rows are copied to x_perm
  void *x_perm;            // [kept rows][d], bf16 (x_bf16) or fp32
  void *x_shared;          // [T][d] or nullptr: every x row again, in token order
  int *shared_off;         // with x_shared: {0, T}, the shared expert's row offsets
  // with x_shared: the shared expert's GEMM plan (one expert of T rows), as
  // launch_expert_plan would write it
  int *shared_mprefix;     // [2]
  int4 *shared_tab1, *shared_tab2;
  int *shared_mdone;       // [ceil(T / kExpertBM) + 1]
  int d, x_bf16;
  int *status;
};
int launch_dispatch(const DispatchArgs &a, cudaStream_t st);
// Expert GEMM plan from offsets: mprefix[n+1] = exclusive scan of
// ceil(M_e / kExpertBM); tab1 / tab2: one int4 per tile of the two GEMMs
// (nblk1 / nblk2 N-blocks): {expert, first row, valid rows, N-block | global
// M-block << 8}, tiles of an expert N-block major, M-block minor; mdone[m] = 0
// for every M-block and mdone[mprefix[n]] = 0 (the expert kernel's GEMM1 ->
// GEMM2 counters).
int launch_expert_plan(const int *offsets, int n, int *mprefix, int4 *tab1, int nblk1, int4 *tab2,
                       int nblk2, int *mdone, cudaStream_t st);
constexpr int kExpertBN = 256;

struct ExpertArgs {
  const void *x_perm;      // [S][d]
  const int *offsets;      // [n+1]
  const int *mprefix;      // [n+1] exclusive scan of ceil(M_e / kExpertBM)
  int4 *tab1, *tab2;       // tile tables of GEMM1 / GEMM2
  int *mdone;              // [M-blocks + 1] GEMM1 -> GEMM2 counters (zeroed by the plan)
  int plan_ready;          // 1: mprefix and the tables were written by the dispatch
  const char *name;        // trace name, or nullptr for the default
  int n, d, f, S;
  const void *W1, *W2;
  const float *b1, *b2;
  void *hid;               // [S][f]
  void *y_perm;            // [S][d]
  int *status;
  // backward (activation gradients, bf16 only): x_perm = dy_perm [S][d],
  // hid = dhid [S][f] (written, then read), y_perm = dx_perm [S][d],
  // mask = the forward's hid [S][f]; W1, W2 the forward's weights; no biases
  int backward;
  const void *mask;
};
int launch_expert_bf16(const ExpertArgs &a, cudaStream_t st);
// moe_test_expert_wait: the GEMM2 tiles' wait limit (0: the default) and an
// M-block whose GEMM1 tiles do not publish (-1: none), for later launches
void set_expert_wait(unsigned long long limit_ns, int withhold_mblock);
int launch_expert_f32(const ExpertArgs &a, cudaStream_t st);

// y_shared [T][d] (expert dtype) or nullptr: the shared expert's rows, added
// to every token before its routed slots
int launch_combine(const void *y_perm, int bf16, const float *gate, const int *row_of,
                   const float *x, int passthrough, int T, int k, int d, float *y,
                   const void *y_shared, cudaStream_t st);
// FP32 FMA throughput probe: blocks x 256 threads, 256 FLOP per thread per iteration
int launch_fma_probe(float *out, int blocks, int iters, int packed, cudaStream_t st);
// *seed += 1 (one thread)
int launch_noise_step(unsigned long long *seed, cudaStream_t st);
int launch_sel_bias_update(const int *counts, int n, int T, int k, float gamma, float *bias,
                           cudaStream_t st);

// ---- backward pass (backward.cu, wgrad_tc.cu, grad_gemm.cu)
struct GateBwdArgs {
  int T, n, k;
  const float *c, *s;          // [T][n] clean logits, Softplus(x W_noise) of the forward
  const int *idx;              // [T][k] kept experts, larger H first
  const float *gate, *dgate;   // [T][k] gates and dL/dgate
  const float *lam_imp, *lam_load, *sw_coef;  // [n] (bwd_coef)
  const int4 *kth;             // [T] {H of the (k+1)-th, its id, H of the k-th, its id}
  unsigned long long seed;
  const unsigned long long *seed_dev;  // when set, the noise key is read here at run time
  uint32_t token_base;         // added to the token index in the noise counter
  int router, noise, has_load;
  float *dc, *dz;              // [T][n] outputs (dz: noise only)
  // rows of a hierarchical layer's secondary gates (T = their count): the
  // token of every row (noise counter) and the first row of every group
  // (seg_off [G+1]: noise stream 1 + group, lam_load + group * n); both
  // nullptr for token rows.  lam_imp may be nullptr (folded into dgate).
  const int *row_token, *seg_off;
  int G;
};
// hierarchical backward (backward_hier.cu)
int launch_hier_coef(const float *lam_load, const float *load_p, const float *load2,
                     const int *cnt, int a, int b, float *lam_p, float *lam_s, cudaStream_t st);
int launch_hier_split(int T, int k1, int k2, int K, int n, const float *pgate,
                      const int *grow, const int *topk_idx, const float *dgate,
                      const float *gate2, const float *lam_imp, float *dgp, float *dgs,
                      cudaStream_t st);
int launch_hier_gate_wgrad(const float *x, int d, const int *row_token, const int *seg_off, int a,
                           int b, const float *dc2, const float *dz2, float *dWg2, float *dWn2,
                           float *dbg2, cudaStream_t st);
int launch_hier_gate_dgrad(const float *dc2, const float *dz2, const float *Wg2, const float *Wn2,
                           const int *seg_off, const int *seg_mblk, int mblk_upper, int a, int d,
                           int b, float *dxs, int T, int k1, const int *grow, float *dx,
                           cudaStream_t st);
int launch_bwd_coef(const float *importance, const float *load, const int *counts, int n, int T,
                    float w_imp, float w_load, float alpha, int router, int noise, float *lam_imp,
                    float *lam_load, float *sw_coef, cudaStream_t st);
// bf16: the expert rows (y_perm, dy_perm, dy_shared / dx_perm, dx_shared)
// are bf16, else fp32
int launch_combine_bwd(const float *dy, const float *gate, const int *row_of, const void *y_perm,
                       int bf16, int T, int k, int d, void *dy_perm, float *dgate, void *dy_shared,
                       cudaStream_t st);
int launch_dx_gather(const void *dx_perm, int bf16, const int *row_of, const float *dy,
                     int passthrough, int T, int k, int d, const void *dx_shared, float *dx,
                     cudaStream_t st);
// fp32 experts' backward: block per expert, gradients written whole (zeroed
// first); db1, db2 may be nullptr
int launch_expert_bwd_f32(const float *x_perm, const float *dy_perm, const int *offsets, int n,
                          int d, int f, const float *W1, const float *b1, const float *W2,
                          float *dx_perm, float *dW1, float *db1, float *dW2, float *db2,
                          const char *name, cudaStream_t st);
int launch_bias_grad(const void *dy_perm, const void *dhid, const int *offsets, int n, int d,
                     int f, float *db2, float *db1, const char *name, cudaStream_t st);
int launch_gate_bwd(const GateBwdArgs &a, cudaStream_t st);
// dc[t][i] += (w_z 2 c_i + w_entropy p_i (log p_i + H_t)) / T, p = softmax(c_t)
int launch_gate_stats_bwd(const float *c, int T, int n, float w_z, float w_entropy, float *dc,
                          cudaStream_t st);
int colsum_parts(int R, int N);
int launch_colsum(const float *X, int R, int N, float *part, float *out, cudaStream_t st);
// weight gradients of the experts on the tensor cores, per expert e with rows
// offsets[e] .. offsets[e+1]-1: dW2_e = dy_perm_e^T hid_e ([d][f]) and
// dW1_e = dhid_e^T x_perm_e ([f][d]), fp32
struct WgradArgs {
  const void *dy_perm, *hid, *dhid, *x_perm;  // [S][d], [S][f], [S][f], [S][d] bf16
  const int *offsets;                         // [n+1]
  int n, d, f, S;
  float *dW1, *dW2;
  int *status;
  const char *name;
};
int launch_wgrad_bf16(const WgradArgs &a, cudaStream_t st);
// C[M][N] = sum_k A(m,k) B(k,n) (+ C when accumulate), fp32; A(m,k) =
// A[m*lda+k] or, with at, A[k*lda+m]; B(k,n) = B[k*ldb+n] or, with bt,
// B[n*ldb+k].  nprob = 2: two problems in one launch, C[p] = A[p] B[p];
// ksum: one problem, C[0] = A[0] B[0] + A[1] B[1].  part: split-K scratch of
// nprob*splits*M*N floats (nullptr: no split).  A, B 16-byte aligned.
struct SgemmArgs {
  int M, N, K;
  const float *A[2];
  const float *B[2];
  float *C[2];
  int lda, ldb, ldc, at, bt;
  int nprob, ksum, accumulate;
  float *part;
  int splits;
  const char *name;
  // Grouped (seg_off set, no split-K): G problems over row segments
  // [seg_off[g], seg_off[g+1]).  seg_k = 1: the segment is the K range (A
  // stored [K][M] with its rows gathered through a_row, B's rows the
  // segment's), C_g = C + g * sC.  seg_k = 0: the segment is the M range (M
  // tiles found through seg_mblk, the exclusive scan of ceil(rows / 128)), A's
  // and C's rows the segment's, B_g = B + g * sB.
  const int *seg_off, *seg_mblk, *a_row;
  int G, seg_k, mblk_upper;
  int64_t sB, sC;
};
int launch_sgemm(const SgemmArgs &a, cudaStream_t st);
int sgemm_splits(int M, int N, int K, int nprob);  // split-K factor for nprob problems of M x N

int launch_importance(const float *gate_sorted, const int *ucoff, int n, float *importance,
                      cudaStream_t st);
// rstats [2] or nullptr: the router statistics' sums over tokens (losses[8],
// [9] become their means; 0 without them)
// dropped (optional): the dropped slots counted elsewhere, instead of counts vs C
int launch_losses(const float *importance, const float *load, const int *counts,
                  const float *prob_sum, int n, int T, int k, int64_t C, int router,
                  float w_imp, float w_load, float alpha, const float *rstats, float *losses,
                  cudaStream_t st, const float *dropped = nullptr);
// dst[i] = src[index[i]] for rows of row_bytes (a multiple of 16); an index
// outside [0, src_rows) gives a zero row and MOE_STATUS_BAD_INDEX
int launch_gather_rows(const void *src, const int *index, void *dst, int64_t rows,
                       int64_t row_bytes, int64_t src_rows, int *status, cudaStream_t st);

}  // namespace moe
