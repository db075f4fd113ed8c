/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of the Sparsely-Gated
 * Mixture-of-Experts layer,  y = sum_i G(x)_i * E_i(x).
 *
 * Library: libmoe_b200.so.  Every entry point is `extern "C"`, takes plain
 * pointers and sizes, returns an int status (MOE_OK = 0, negative = error)
 * and is asynchronous on the given CUDA stream.
 *
 * Sources (page title, section), cited per entry point below:
 *  [SGMoE-note] "Outrageously Large Neural Networks: The Sparsely-Gated
 *               Mixture-of-Experts Layer" reading note (chenshi221.pages.dev),
 *               "Sparsely-Gated MoE 层架构", "Noisy Top-K Gating", "负载均衡",
 *               "分层 MoE".
 *  [SGMoE-xyz]  "極大規模神經網路：稀疏門控專家混合層" (xyznot.com, arXiv
 *               1701.06538), "方法（與關鍵公式）": "Noisy Top-K 門控",
 *               "負載平衡損失".
 *  [MoE-deep]   "MoE 稀疏架构深度解析" (tufusi.com), §3.1 核心架构,
 *               §3.2 负载均衡问题.
 *
 * Conventions shared by every call
 *  - Memory ownership: every pointer argument is caller-owned DEVICE memory
 *    (the moe_config / parameter structs themselves are host memory and are
 *    read during the call only).  The library allocates nothing; scratch
 *    space is the caller's workspace `ws` of at least
 *    moe_workspace_size() bytes, 256-byte aligned.
 *  - Layouts are row-major.  x is [T][d] fp32.  Gate weights are stored as in
 *    the pages' x*W products: W_g, W_noise are [d][n] fp32.  Expert weights
 *    are stored K-major, as each linear map's [out][in]: W1 is [n][f][d],
 *    W2 is [n][d][f], bf16 (MOE_BF16) or fp32 (MOE_F32); biases b1 [n][f],
 *    b2 [n][d] are fp32 and may be NULL (zero).
 *  - Alignment: every array pointer must be 16-byte aligned; d and f must be
 *    multiples of 8.
 *  - Routing slots: topk_idx / topk_gate are [T][k]; slot j of a token holds
 *    its j-th largest noisy logit (ties: lower expert index first).
 *  - Errors: argument problems are found on the host before any launch and
 *    returned as MOE_EINVAL / MOE_EWORKSPACE; a failed launch returns
 *    MOE_ECUDA.  Problems that only the device can see (a NaN logit, an
 *    expert id out of range, a bounded wait that ran out) are OR-ed into the
 *    caller's device word `*status` as MOE_STATUS_* bits; no kernel ever
 *    traps.  The library never clears *status: the caller zeroes it and reads
 *    it after synchronising.
 *  - Determinism: for fixed inputs every output is bitwise reproducible
 *    (fixed-order reductions, stable permutation).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point is exported from the shared library. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *moe_stream_t;

enum {
  MOE_OK = 0,
  MOE_EINVAL = -1,      /* invalid configuration or NULL required pointer */
  MOE_EWORKSPACE = -2,  /* workspace smaller than moe_workspace_size()    */
  MOE_ECUDA = -3,       /* a CUDA call or kernel launch failed            */
  MOE_EDEVICE = -4      /* no usable sm_100 device                        */
};

enum { MOE_ROUTER_NOISY_TOPK = 0, MOE_ROUTER_SWITCH = 1, MOE_ROUTER_SIGMOID = 2 };
enum { MOE_F32 = 0, MOE_BF16 = 1 };
/* How the gate's fp32 projections x W_g, x W_noise are computed:
 * MOE_GATE_FP32   fp32 fused multiply-adds on the CUDA cores;
 * MOE_GATE_TF32X3 tensor cores with a three-pass TF32 split (hi*hi + hi*lo +
 *                 lo*hi, hi = nearest tf32, lo = remainder), fp32 accumulation:
 *                 about the accuracy of fp32 multiply-adds, several times faster. */
enum { MOE_GATE_FP32 = 0, MOE_GATE_TF32X3 = 1 };

/* bits OR-ed into *status by the kernels */
enum {
  MOE_STATUS_NONFINITE = 1,  /* a gate logit (or its noise scale) was NaN/Inf */
  MOE_STATUS_BAD_INDEX = 2,  /* an expert id outside [0,n) was ignored        */
  MOE_STATUS_TIMEOUT = 4,    /* a bounded on-chip wait gave up; outputs void  */
  MOE_STATUS_OVERFLOW = 8    /* a size exceeded a kernel limit                */
};

/* Layer description.
 *   T tokens, d model width, n experts, k experts per token, f hidden width.
 *   Hierarchical layer ([SGMoE-note] "分层 MoE"): hier_a > 0 groups of hier_b
 *   experts each; the primary gate keeps hier_k1 groups, each group's gate
 *   keeps hier_k2 of its experts; then n = hier_a*hier_b, k = hier_k1*hier_k2.
 *   router: MOE_ROUTER_NOISY_TOPK ([SGMoE-xyz] "Noisy Top-K 門控"),
 *   MOE_ROUTER_SWITCH ([MoE-deep] §3.1: softmax over all experts, top-1, gate
 *   = the winner's probability, no noise) or MOE_ROUTER_SIGMOID ([MoE-deep]
 *   §6.2, §6.3: the k largest routing scores h_i + b_i are kept, b being the
 *   selection bias (moe_gate_params.sel_bias, moe_sel_bias_update); the gates
 *   are Sigmoid(h_i) / sum of Sigmoid(h_j) over the kept j, without the bias;
 *   no noise, flat only).  h = x W_g + b_g as for the other routers.
 *   shared_expert: 1 adds one always-active expert to every token, weight 1
 *   ([MoE-deep] §5.2, §6.2: y = E_shared(x) + sum_j g_j E_j(x)); a token whose
 *   routed slots all overflowed keeps it (pass-through replaces only the
 *   routed sum).  Only moe_forward evaluates it.
 *   router_stats: 1 makes moe_forward report the router z-loss and the gate
 *   entropy ([MoE-intro] "第三部分：MoE 的训练挑战与解决方案") in losses[8], [9]
 *   over the flat (or primary) gate's clean logits h = x W_g + b_g.
 *   noise: 1 adds StandardNormal() * Softplus(x W_noise); the deviate for
 *   (seed, token t, expert i, gate g) comes from Philox4x32-10 with key
 *   (seed lo, seed hi) and counter (t, i/4, g, 0): words 0,1 give the cosine
 *   and sine branches of one Box-Muller transform for experts 4m, 4m+1,
 *   words 2,3 those of a second one for 4m+2, 4m+3; g = 0 for the
 *   flat/primary gate and 1+group for a secondary gate.
 *   capacity_factor > 0 limits every expert to C = ceil(T*k*cf/n) slots
 *   ([MoE-deep] §3.2); slots beyond C (in token order) are dropped.
 *   overflow_passthrough: 1 gives a token whose every slot was dropped the
 *   output y = x (it "goes through the residual", [MoE-deep] §3.2).
 *   w_importance, w_load: weights of the two CV^2 losses ([SGMoE-xyz]
 *   "負載平衡損失"; 0.1 each in [SGMoE-note] "缺点与局限性"); alpha_aux: the
 *   Switch loss coefficient ([MoE-deep] §3.2).  gate_precision: see
 *   MOE_GATE_* ([SGMoE-note] "缺点与局限性": the gate needs fp32). */
typedef struct moe_config {
  int32_t T, d, n, k, f;
  int32_t hier_a, hier_b, hier_k1, hier_k2;
  int32_t router;
  int32_t noise;
  int32_t expert_dtype;       /* MOE_F32 or MOE_BF16 */
  uint64_t seed;
  double capacity_factor;
  int32_t overflow_passthrough;
  float w_importance, w_load, alpha_aux;
  int32_t gate_precision;     /* MOE_GATE_FP32 or MOE_GATE_TF32X3 */
  int32_t shared_expert;      /* 0 or 1 */
  int32_t router_stats;       /* 1: moe_forward reports losses[8], [9] */
  int32_t backward;           /* 1: the workspace also serves moe_backward and
                                 moe_forward keeps what it needs (0 or 1) */
  float w_z, w_entropy;       /* weights of the router z-loss and of the gate
                                 entropy in moe_backward's loss (0: none) */
  int64_t token_base;         /* index of the first token in the noise counter:
                                 0 for a whole batch; a data-parallel shard of a
                                 batch passes its first token's index in the batch,
                                 so that its tokens draw the noise they would draw
                                 in the whole batch (0 <= token_base,
                                 token_base + T <= 2^32) */
} moe_config;

/* Gate parameters.  Flat layer: W_g, W_noise [d][n], b_g [n] (per-expert
 * clean-logit bias, may be NULL).  Hierarchical layer: the same three for the
 * primary gate over hier_a groups, plus the secondary gates W_g2, W_noise2
 * [hier_a][d][hier_b] and b_g2 [hier_a][hier_b] (may be NULL).  W_noise /
 * W_noise2 may be NULL when noise == 0.  sel_bias [n]: the selection bias of
 * MOE_ROUTER_SIGMOID (NULL: zero; ignored by the other routers).
 * seed_dev: NULL, or one uint64 in device memory (8-byte aligned) that then
 * replaces cfg->seed as the noise key: the routing kernel and moe_backward's
 * gate backward read it when they run, so a captured CUDA graph draws the
 * noise of whatever the word holds at each replay.  The pages' noisy gate
 * draws a new StandardNormal() every time it runs ([SGMoE-xyz] "Noisy Top-K
 * 門控"); a caller advances the word once per step with moe_noise_step and
 * leaves it alone between a forward and its backward. */
typedef struct moe_gate_params {
  const float *W_g, *b_g, *W_noise;
  const float *W_g2, *b_g2, *W_noise2;
  const float *sel_bias;
  const uint64_t *seed_dev;
} moe_gate_params;

/* Expert parameters: W1 [n][f][d], W2 [n][d][f] of expert_dtype; b1 [n][f],
 * b2 [n][d] fp32 or NULL.  With shared_expert: the shared expert's W1s [f][d],
 * W2s [d][f] (expert_dtype), b1s [f], b2s [d] (fp32 or NULL); else unused. */
typedef struct moe_expert_params {
  const void *W1;
  const float *b1;
  const void *W2;
  const float *b2;
  const void *W1s;
  const float *b1s;
  const void *W2s;
  const float *b2s;
} moe_expert_params;

/* Text for a return code. */
MOE_API const char *moe_strerror(int code);

/* Validates cfg.  MOE_OK or MOE_EINVAL.  Limits: T >= 0, 1 <= k <= min(n,8),
 * 1 <= n <= 8192, d, f multiples of 8, d <= 16384, f <= 65536; Switch router:
 * k = 1, no noise, n <= 4096, flat only; sigmoid router: no noise, flat only;
 * shared_expert 0 or 1. */
MOE_API int moe_validate(const moe_config *cfg);

/* Expert capacity C = ceil(T*k*capacity_factor/n), or INT64_MAX when
 * capacity_factor <= 0 ([MoE-deep] §3.2: C = tokens per batch / E * factor;
 * with k slots per token the routed slots are T*k). */
MOE_API int moe_capacity(const moe_config *cfg, int64_t *C);

/* Bytes of workspace that every call below accepts for this cfg (the same
 * number for every entry point; moe_forward needs all of it). */
MOE_API int moe_workspace_size(const moe_config *cfg, size_t *bytes);

/* ---------------------------------------------------------------- steps */

/* Gate: H(x)_i = (x W_g)_i + b_g,i + StandardNormal()*Softplus((x W_noise)_i),
 * KeepTopK(H, k), G(x) = Softmax(KeepTopK(H, k))  ([SGMoE-xyz] "Noisy Top-K
 * 門控"; [SGMoE-note] "Noisy Top-K Gating"); Switch router per [MoE-deep]
 * §3.1; hierarchical gate per [SGMoE-note] "分层 MoE" (slot ps*k2+ss holds
 * expert g*b+j with gate G_p(x)_g * G_g(x)_j, g the ps-th kept group).
 * Outputs: topk_idx [T][k] int32, topk_gate [T][k] fp32,
 *   load [n]: the smoothed load Load(X)_i = sum_x P(x,i),
 *     P(x,i) = Phi(((x W_g)_i - kth_excluding(H(x),k,i)) / Softplus((x W_noise)_i))
 *     ([SGMoE-xyz] "負載平衡損失"); without noise its zero-noise limit, the
 *     number of tokens that keep expert i.  Hierarchical: Load_p(X)_g *
 *     Load_g(X_g)_j / |X_g| for expert g*b+j, 0 for an empty group.
 *   prob_sum [n] (may be NULL): sum over tokens of the Switch router's
 *     softmax (zeros for the noisy gate).
 * Errors: MOE_EINVAL for a NULL x / W_g / outputs (or W_noise with noise on,
 * W_g2 for a hierarchical cfg). */
MOE_API int moe_gate(const moe_config *cfg, const float *x, const moe_gate_params *gp,
             int32_t *topk_idx, float *topk_gate, float *load, float *prob_sum,
             void *ws, size_t ws_bytes, int32_t *status, moe_stream_t stream);

/* Dispatch: E_i(x) is only evaluated where G(x)_i != 0 ([SGMoE-note]
 * "Sparsely-Gated MoE 层架构"), so every (token, slot) pair goes to its
 * expert.  Pairs are taken in (token, slot) order; the r-th pair of expert e
 * is kept iff r < C ([MoE-deep] §3.2) and lands in row offsets[e] + r.
 * Outputs: counts [n] (pairs per expert before the capacity cut), offsets
 * [n+1] (exclusive scan of min(count, C)), perm_token [T*k] (token of every
 * kept row; rows >= offsets[n] untouched), row_of [T][k] (row of a kept
 * pair, -1 if dropped or its id was out of range -- the latter also sets
 * MOE_STATUS_BAD_INDEX), x_perm [T*k][d] (x rows gathered into the kept rows,
 * cast to expert_dtype; may be NULL together with x to skip the gather). */
MOE_API int moe_dispatch(const moe_config *cfg, const float *x, const int32_t *topk_idx,
                 int32_t *counts, int32_t *offsets, int32_t *perm_token,
                 int32_t *row_of, void *x_perm, void *ws, size_t ws_bytes,
                 int32_t *status, moe_stream_t stream);

/* Allocation-free variant of moe_dispatch.  The pages have no counterpart:
 * this entry point exists for callers that are given only their input and
 * output buffers and cannot obtain scratch device memory -- e.g. a plugin of
 * a host inference engine that plans all memory up front and passes no
 * allocator, or a serving loop that must not call cudaMalloc after start-up
 * (it synchronises the device and can fail under memory pressure).
 * Same arguments, outputs and status bits as moe_dispatch, without ws.  Its
 * scratch (per-block histograms and their scanned bases, uncapped offsets,
 * one counter) takes 2*B*n + n + 2 int32, B = ceil(T / t) dispatch blocks of t tokens,
 * t = T/296 rounded up to a multiple of 32 and clamped to [32, 256].  It
 * lives in one fixed device array of MOE_DISPATCH_NOALLOC_SCRATCH_INTS int32
 * (4 MiB) that every GPU loading the library keeps until the process exits.
 * A call needing more returns MOE_EWORKSPACE before any device work (n = 256
 * experts fit up to T = 524032 tokens, n = 4096 up to T = 4064).  The first
 * call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current), so make that first call before any stream
 * capture.  All calls share the array: every element a call reads is written
 * earlier in the same call, so results never depend on earlier calls, but
 * calls that overlap on the GPU (other streams, unordered host threads) race
 * on it.  It calls no allocator. */
#define MOE_DISPATCH_NOALLOC_SCRATCH_INTS (1 << 20)
MOE_API int moe_dispatch_noalloc(const moe_config *cfg, const float *x,
                                 const int32_t *topk_idx, int32_t *counts,
                                 int32_t *offsets, int32_t *perm_token, int32_t *row_of,
                                 void *x_perm, int32_t *status, moe_stream_t stream);

/* Expert FFN on the expert-contiguous rows: rows offsets[e] .. offsets[e+1]-1
 * of x_perm go through expert e ([SGMoE-note] "Sparsely-Gated MoE 层架构":
 * one hidden ReLU layer):  y_perm = ReLU(x_perm W1_e^T + b1_e) W2_e^T + b2_e.
 * bf16 experts: bf16 operands, fp32 accumulation (tcgen05 tensor cores), the
 * hidden layer rounded to bf16, y_perm written as bf16.  fp32 experts: fp32
 * throughout.  x_perm, y_perm: [T*k][d] of expert_dtype. */
MOE_API int moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                   const moe_expert_params *ep, void *y_perm, void *ws,
                   size_t ws_bytes, int32_t *status, moe_stream_t stream);

/* Combine: y_t = sum_j topk_gate[t][j] * y_perm[row_of[t][j]] over the kept
 * slots j (in slot order) ([SGMoE-note] "Sparsely-Gated MoE 层架构": y = sum_i
 * G(x)_i E_i(x)).  A dropped slot adds nothing (gates are not renormalised);
 * with overflow_passthrough a token with no kept slot gets y_t = x_t
 * ([MoE-deep] §3.2), otherwise 0.  y: [T][d] fp32; x may be NULL without
 * pass-through. */
MOE_API int moe_combine(const moe_config *cfg, const void *y_perm, const float *topk_gate,
                const int32_t *row_of, const float *x, float *y, int32_t *status,
                moe_stream_t stream);

/* Balancing statistics ([SGMoE-xyz] "負載平衡損失"; [MoE-deep] §3.2).
 * importance [n]: Importance(X)_i = sum_x G(x)_i.
 * losses [10]:
 *   [0] L_importance = w_importance * CV(Importance)^2
 *   [1] L_load       = w_load * CV(load)^2
 *   [2] N * sum_i f_i P_i  (Switch: f_i = counts_i / T before the capacity
 *       cut, P_i = prob_sum_i / T); 0 for the noisy and sigmoid routers
 *   [3] alpha_aux * [2]
 *   [4] dropped slots / (T*k),   [5] CV(Importance)^2,   [6] CV(load)^2,
 *   [7] dropped slots
 *   [8] router z-loss: mean over tokens of |h|^2, the squared L2 norm of the
 *       clean logits (our reading of "penalise the L2 norm of the logits
 *       before the softmax"); [9] mean over tokens of the entropy of
 *       softmax(h) over all experts (a statistic; the "gate entropy loss"
 *       rewards it, so its weight is negative).  Both come from moe_forward
 *       with router_stats = 1 and are 0 otherwise (moe_balance_losses always
 *       writes 0 there).
 * CV^2 is the population variance over the squared mean (0 for a zero
 * mean), evaluated in fp64.  counts and load come from moe_dispatch /
 * moe_gate; prob_sum may be NULL for the noisy gate. */
MOE_API int moe_balance_losses(const moe_config *cfg, const int32_t *topk_idx,
                       const float *topk_gate, const int32_t *counts,
                       const float *load, const float *prob_sum, float *importance,
                       float *losses, void *ws, size_t ws_bytes, int32_t *status,
                       moe_stream_t stream);

/* Selection-bias update of MOE_ROUTER_SIGMOID ([MoE-deep] §6.3): with
 * counts [n] from a dispatch of T tokens (before the capacity cut), an expert
 * that took more than the average T*k/n slots gets sel_bias -= gamma, one that
 * took fewer gets sel_bias += gamma (fp32), one exactly at the average keeps
 * its bias; the comparison is exact (counts*n against T*k).  sel_bias [n] is
 * read and written in place on the stream.  Errors: MOE_EINVAL for NULL
 * pointers or an invalid cfg. */
MOE_API int moe_sel_bias_update(const moe_config *cfg, const int32_t *counts, float gamma,
                                float *sel_bias, moe_stream_t stream);

/* Adds 1 to the device word *seed_dev (see moe_gate_params.seed_dev) in
 * stream order, so that the next moe_forward / moe_gate on the stream draws
 * fresh noise ([SGMoE-xyz] "Noisy Top-K 門控": a new StandardNormal() per
 * evaluation).  One single-thread kernel; capturable in a CUDA graph.
 * Errors: MOE_EINVAL for a NULL or misaligned pointer, MOE_ECUDA. */
MOE_API int moe_noise_step(uint64_t *seed_dev, moe_stream_t stream);

/* ---------------------------------------------------------------- fused */

/* The whole layer on one stream: gate, dispatch, experts (and the shared
 * expert when cfg->shared_expert), combine and the balancing statistics,
 * every intermediate in ws.  Outputs as the step calls above: y [T][d],
 * topk_idx, topk_gate [T][k], importance, load [n], counts [n], losses [10]. */
MOE_API int moe_forward(const moe_config *cfg, const float *x, const moe_gate_params *gp,
                const moe_expert_params *ep, float *y, int32_t *topk_idx,
                float *topk_gate, float *importance, float *load, int32_t *counts,
                float *losses, void *ws, size_t ws_bytes, int32_t *status,
                moe_stream_t stream);

/* ---------------------------------------------------------------- expert parallel */

/* Row gather for the expert-parallel layer ([MoE-deep] §7.1: each token's
 * rows travel to the device of their expert and back).  dst row i = src row
 * index[i], i < rows, each row row_bytes long (a positive multiple of 16);
 * src holds src_rows rows.  An index outside [0, src_rows) gives a zero row
 * and sets MOE_STATUS_BAD_INDEX.  src, dst: device memory, 16-byte aligned,
 * not overlapping; index [rows] int32 device memory.  Used to regroup rows
 * received from every rank by local expert before moe_expert_ffn, and (with
 * the inverse index) to put the results back in the exchange's order.
 * Errors: MOE_EINVAL (NULL or misaligned pointers, a bad row_bytes, negative
 * sizes), MOE_EDEVICE, MOE_ECUDA. */
MOE_API int moe_gather_rows(const void *src, const int32_t *index, void *dst, int64_t rows,
                            int64_t row_bytes, int64_t src_rows, int32_t *status,
                            moe_stream_t stream);

/* The balancing losses of a batch split over data-parallel shards, from its
 * totals ([SGMoE-xyz] "負載平衡損失"; [MoE-deep] §3.2): importance, load,
 * counts and (Switch) prob_sum [n] are the sums over all shards' tokens,
 * dropped [1] the sum of the slots each shard's own capacity cut dropped;
 * cfg->T is the whole batch's token count.  losses[0..7] as moe_balance_losses
 * (losses[4] = dropped / (T*k), losses[7] = dropped), losses[8], [9] = 0.
 * Errors: MOE_EINVAL (invalid cfg, NULL pointers; prob_sum for Switch),
 * MOE_EDEVICE, MOE_ECUDA. */
MOE_API int moe_balance_from_totals(const moe_config *cfg, const float *importance,
                                    const float *load, const int32_t *counts,
                                    const float *prob_sum, const float *dropped, float *losses,
                                    int32_t *status, moe_stream_t stream);

/* ---------------------------------------------------------------- backward */

/* Gradients written by moe_backward, fp32, caller-owned device memory in the
 * layouts of the parameters.  Any pointer may be NULL (that gradient is not
 * written) except dW1 and dW2; dW_noise is ignored without noise, the shared
 * expert's without a shared expert.  dgate [T][k] and dlogits [T][n] are
 * optional intermediate results: dL/d topk_gate and dL/d(x W_g + b_g). */
typedef struct moe_grads {
  float *dW_g, *db_g, *dW_noise;        /* [d][n], [n], [d][n]; hierarchical: the primary
                                           gate's [d][hier_a], [hier_a], [d][hier_a] */
  float *dW1, *db1, *dW2, *db2;         /* [n][f][d], [n][f], [n][d][f], [n][d] */
  float *dW1s, *db1s, *dW2s, *db2s;     /* [f][d], [f], [d][f], [d] */
  float *dgate, *dlogits;               /* [T][k], [T][n] (dlogits: flat layers only) */
  float *dW_g2, *db_g2, *dW_noise2;     /* hierarchical: the secondary gates'
                                           [hier_a][d][hier_b], [hier_a][hier_b],
                                           [hier_a][d][hier_b] */
} moe_grads;

/* Backward pass of the layer (flat or hierarchical).  The pages give no
 * backward formulas; they fix which paths carry a gradient: the kept gates
 * are a smooth function of the logits ([SGMoE-xyz] "常見問題"), KeepTopK
 * gives the experts it drops none ([SGMoE-note] "缺点与局限性"), and the
 * noise lets the load loss reach the gate through Phi ([SGMoE-note] "Noisy
 * Top-K Gating").  Computes the gradients of
 *   L = sum(dy * y) + losses[0] + losses[1] + losses[3]
 *       + w_z * losses[8] - w_entropy * losses[9]
 * (dy [T][d] fp32, the upstream gradient of moe_forward's y, plus the
 * weighted balancing losses; the router z-loss mean_t |h_t|^2 and the gate
 * entropy mean_t H(softmax(h_t)) of [MoE-intro] "第三部分" enter with the
 * weights w_z and -w_entropy, so a positive w_entropy rewards entropy) with
 * respect to x (dx [T][d], fp32, written) and
 * every parameter (grads).  With bf16 experts (mixed precision) the gradients
 * reaching the expert rows (g * dy), the hidden layer and the expert inputs
 * are kept in bf16 as the forward keeps its activations, accumulation is
 * fp32; with fp32 experts everything is fp32.  The gate is fp32 throughout.  The selection bias of MOE_ROUTER_SIGMOID gets no
 * gradient (it enters only the choice of experts).
 *
 * Preconditions: cfg->backward == 1 and ws is the workspace of the preceding
 * moe_forward with the same cfg, x and parameters, whose outputs topk_idx,
 * topk_gate, importance, load and counts are passed back here; both calls
 * on the same stream, in that order.  ws is read and overwritten.
 * Hierarchical layer ([SGMoE-note] "分层 MoE"): the slot gate G_p(x)_g G_g(x)_j
 * passes dL/dG_p = sum over its slots of dL/dslot G_g and dL/dG_g = dL/dslot
 * G_p to the two levels; Load(g*b+j) = Load_p_g Load_g_j / |X_g| (the
 * forward's reading, |X_g| a count) sends the load loss to both levels; each
 * level's gate then takes the flat gate's chain rule, a secondary row with
 * its own noise stream (gate 1 + g).  grads->dW_g, db_g, dW_noise are the
 * primary gate's, dW_g2, db_g2, dW_noise2 the secondary gates'; dlogits is
 * not written.  No shared expert with a hierarchical layer.
 * Errors: MOE_EINVAL for cfg->backward != 1, a hierarchical layer with a shared expert, NULL required pointers or misaligned ones (x, dy, dx 16-byte
 * aligned); MOE_EWORKSPACE; MOE_ECUDA.  Device-side timeouts are OR-ed into
 * *status (MOE_STATUS_TIMEOUT). */
MOE_API int moe_backward(const moe_config *cfg, const float *x, const moe_gate_params *gp,
                         const moe_expert_params *ep, const float *dy, const int32_t *topk_idx,
                         const float *topk_gate, const float *importance, const float *load,
                         const int32_t *counts, float *dx, const moe_grads *grads, void *ws,
                         size_t ws_bytes, int32_t *status, moe_stream_t stream);

/* ---------------------------------------------------------------- measurement */

/* FP32 FMA throughput probe (a measurement helper; the pages have no
 * counterpart).  Launches `blocks` blocks of 256 threads; every thread runs
 * 16 independent fp32 FMA chains for iters x 8 steps, i.e. 256 FLOP per
 * thread per iteration, blocks * 256 * iters * 256 FLOP in all, and writes
 * one float per thread to out[blocks * 256] (device memory).  packed = 0
 * issues scalar fma.rn.f32, packed = 1 the two-wide fma.rn.f32x2.  Timing it
 * with CUDA events gives the FP32 FMA peak that bounds the fp32 gate GEMM.
 * Errors: MOE_EINVAL (NULL out, blocks or iters < 1), MOE_ECUDA. */
MOE_API int moe_fma_probe(float *out, int blocks, int iters, int packed, moe_stream_t stream);

/* Test hook for the expert kernel's bounded cross-CTA wait (failure
 * detection; the pages have no counterpart).  In the fused expert kernel a
 * GEMM2 tile waits for the GEMM1 tiles of its 128-row M-block to publish
 * their hidden rows; the wait gives up after a limit (default 2 s), sets
 * MOE_STATUS_TIMEOUT in *status, and the kernel drains its copies and MMAs
 * (bounded), frees its tensor memory and returns, leaving the context
 * usable.  moe_test_expert_wait(limit_ns, withhold_mblock) sets, for the
 * expert launches that follow in this process, that limit (0: back to the
 * default) and one M-block whose GEMM1 tiles skip their publish
 * (withhold_mblock = -1: none), so that the wait for it can only end by its
 * limit; the outputs of such a call are void.  Process-wide, not for
 * concurrent use; reset with (0, -1).  Always MOE_OK. */
MOE_API int moe_test_expert_wait(unsigned long long limit_ns, int withhold_mblock);

/* ---------------------------------------------------------------- tracing */

/* Per-kernel timing with CUDA events recorded around every launch on its own
 * stream.  Off by default.  moe_trace_count/get synchronise on the recorded
 * events and report, per kernel name, the launches and total milliseconds
 * since the last reset.  moe_launch_count counts every kernel the library
 * launched since load (tracing on or off).  Not thread-safe. */
MOE_API int moe_trace_enable(int on);
MOE_API int moe_trace_reset(void);
MOE_API int moe_trace_count(void);
MOE_API int moe_trace_get(int i, const char **name, int *launches, double *total_ms);
MOE_API long long moe_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
