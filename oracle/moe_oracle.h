/*
 * moe_oracle.h -- plain single-threaded CPU oracle for the forward and backward
 * passes of the Sparsely-Gated Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This code exists to check the CUDA path; it is
 * never part of the product path.  Only tests/, the smoke check and the
 * bench's CPU-baseline leg may load it.  It shares no source, header, table or
 * helper with the CUDA library: every formula below is written out again from
 * the pages it cites.
 *
 * Arithmetic: fp64 accumulation everywhere (the backward's bf16 mode rounds
 * where the mixed-precision kernels store, see orc_backward).  Two results are
 * deliberately taken in fp32 because an integer decision hangs on them and
 * the kernel takes that decision in fp32: the gate logits H used for
 * KeepTopK / argmax.
 *
 * Sources (page title, section):
 *  [SGMoE-note]  "Outrageously Large Neural Networks: The Sparsely-Gated
 *                Mixture-of-Experts Layer" reading note (chenshi221.pages.dev),
 *                sections "Sparsely-Gated MoE 层架构", "Noisy Top-K Gating",
 *                "负载均衡", "分层 MoE", "缺点与局限性".
 *  [SGMoE-xyz]   "極大規模神經網路：稀疏門控專家混合層" (xyznot.com, arXiv
 *                1701.06538), section "方法（與關鍵公式）": "Noisy Top-K 門控" and
 *                "負載平衡損失".
 *  [MoE-intro]   "MoE (Mixture-of-Experts) 算法介绍" (wkbse.com), "工作流程";
 *                "第三部分：MoE 的训练挑战与解决方案" (router z-loss, gate
 *                entropy loss).
 *  [MoE-deep]    "MoE 稀疏架构深度解析" (tufusi.com), §3.1 核心架构,
 *                §3.2 负载均衡问题, §5.2 DeepSeekMoE 的细粒度设计 (shared
 *                expert), §6.2 DeepSeek-V3 的 MoE 配置 (sigmoid scores
 *                normalised over the top K), §6.3 Auxiliary-Loss-Free 负载均衡
 *                (selection bias and its update).
 *  [Philox]      Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
 *                as 1, 2, 3", SC'11 (Philox4x32-10).
 *  [Box-Muller]  Box & Muller, "A note on the generation of random normal
 *                deviates", Ann. Math. Stat. 1958.
 *
 * Parity pins for every function are in tests/test_oracle_*.py.  Parity
 * unpinned: the exact form of the hierarchical Load (the pages give the
 * structure of the two-level gate but no formula for its balancing losses);
 * it is pinned only through its zero-noise limit.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer description.  Flat layer: hier_a == 0.  Hierarchical layer: the
 * primary gate picks hier_k1 of hier_a groups, each group's secondary gate
 * picks hier_k2 of hier_b experts; then n must be hier_a*hier_b and
 * k == hier_k1*hier_k2. */
typedef struct {
  int T, d, n, k, f;
  int hier_a, hier_b, hier_k1, hier_k2;
  int router;               /* 0: noisy top-k softmax gate; 1: Switch top-1 router;
                               2: sigmoid scores, top k of score + selection bias,
                               gates normalised over the kept k (no noise) */
  int noise;                /* 1: add StandardNormal * Softplus(x W_noise)        */
  uint64_t seed;
  double capacity_factor;   /* <= 0: no capacity limit                           */
  int passthrough;          /* 1: a token whose every slot overflowed gets y = x  */
  int expert_bf16;          /* 1: expert weights and activations are bf16         */
  double w_importance, w_load, alpha;
  int shared_expert;        /* 1: y also gets one always-active expert, weight 1 */
  int router_stats;         /* 1: losses[8], [9] get the router z-loss and entropy */
  double w_z, w_entropy;    /* weights of the z-loss and of the entropy in the
                               backward's loss (orc_backward) */
} orc_cfg;

/* ---- noise ------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
double orc_box_muller(uint32_t w0, uint32_t w1, int branch);
double orc_noise(uint64_t seed, uint32_t token, uint32_t expert, uint32_t gate_id);

/* ---- small helpers with a closed form ---------------------------------- */
double orc_softplus(double z);
double orc_phi(double z);
double orc_cv2(const double *v, int n);
float  orc_bf16_round(float v);
int64_t orc_capacity(int T, int k, int n, double capacity_factor);

/* ---- gate, one token (one row of the batch) ---------------------------- */
/* x[d]; Wg, Wn: [d][n] row-major; bg: [n] or NULL; Wn may be NULL when noise
 * is off.  Writes c[n] = (x Wg)+bg, s[n] = Softplus(x Wn) (0 if noise off),
 * H[n] (fp32: the score KeepTopK ranks; for router 2 it is c + sel_bias),
 * order[n] = indices sorted by (H desc, index asc), gates[k] (softmax over
 * the kept k for router 0; the full-softmax probability of the argmax for
 * router 1, k must be 1; for router 2 Sigmoid(c_i) over the sum of
 * Sigmoid(c_j) of the kept k) and, for router 1, p[n] (may be NULL).
 * sel_bias [n] (router 2 only) may be NULL. */
void orc_gate_row(int d, int n, int k, int router, int noise, uint64_t seed,
                  uint32_t token, uint32_t gate_id, const float *x,
                  const float *Wg, const float *bg, const float *Wn,
                  double *c, double *s, float *H, int *order, double *gates,
                  double *p, const float *sel_bias);

/* Selection-bias update of router 2 ([MoE-deep] §6.3): an expert that took
 * more than the average T*k/n slots (counts before capacity) gets
 * bias -= gamma, one that took fewer gets bias += gamma, in fp32. */
void orc_sel_bias_update(int n, int T, int k, const int32_t *counts, float gamma, float *bias);

/* P(x,i) of the smoothed load estimator for every i, from one token's c, s
 * and H (as written by orc_gate_row). */
void orc_load_row(int n, int k, int noise, const double *c, const double *s,
                  const float *H, double *P);

/* ---- dispatch: stable expert-major permutation with capacity ------------ */
/* idx[T][k] (any value outside [0,n) is ignored and counted in *n_invalid).
 * counts[n] (before capacity), offsets[n+1] (exclusive scan of min(count,C)),
 * perm_token/perm_slot[offsets[n]], row_of[T][k] (-1: dropped or invalid). */
void orc_dispatch(int T, int k, int n, int64_t C, const int32_t *idx,
                  int32_t *counts, int32_t *offsets, int32_t *perm_token,
                  int32_t *perm_slot, int32_t *row_of, int64_t *n_invalid);

/* ---- one expert applied to one token ----------------------------------- */
/* W1: [f][d], b1: [f], W2: [d][f], b2: [d].  bf16 == 1: W1/W2 hold bf16 bit
 * patterns (uint16), x and the hidden layer are rounded to bf16. */
void orc_expert_row(int d, int f, int bf16, const float *x, const void *W1,
                    const float *b1, const void *W2, const float *b2, double *y);

/* ---- whole forward pass ------------------------------------------------- */
typedef struct {
  const float *x;                /* [T][d]                                    */
  const float *Wg, *bg, *Wn;     /* flat/primary gate: [d][n'] , [n'], [d][n'] */
  const float *Wg2, *bg2, *Wn2;  /* hierarchical secondary gates: [a][d][b], [a][b], [a][d][b] */
  const void *W1; const float *b1;   /* [n][f][d], [n][f] */
  const void *W2; const float *b2;   /* [n][d][f], [n][d] */
  const float *sel_bias;             /* [n] selection bias of router 2, or NULL (0) */
  const void *W1s; const float *b1s; /* shared expert: [f][d], [f] */
  const void *W2s; const float *b2s; /* [d][f], [d] */
} orc_inputs;

typedef struct {
  double *y;            /* [T][d]                                   */
  int32_t *topk_idx;    /* [T][k]                                   */
  double *topk_gate;    /* [T][k]                                   */
  double *importance;   /* [n]                                      */
  double *load;         /* [n]                                      */
  double *prob_sum;     /* [n]   sum over tokens of the router softmax (router 1) */
  int32_t *counts;      /* [n]                                      */
  int32_t *row_of;      /* [T][k]                                   */
  double *losses;       /* [10]  see orc_forward                    */
  float *near_tie;      /* [T]   H_(k) - H_(k+1) of the deciding gate, or NULL */
} orc_outputs;

/* Gate over a whole batch: topk_idx / topk_gate [T][k], load [n],
 * prob_sum [n] (may be NULL), near_tie [T] (may be NULL).  0 or -1. */
int orc_gate_batch(const orc_cfg *cfg, const orc_inputs *in, int32_t *topk_idx,
                   double *topk_gate, double *load, double *prob_sum, float *near_tie);

/* The gate for the tokens listed in tokens[0..ntok-1] (NULL: 0..ntok-1):
 * output row r belongs to token tokens[r] (x row and noise counter). */
int orc_gate_tokens(const orc_cfg *cfg, const orc_inputs *in, const int32_t *tokens, int ntok,
                    int32_t *topk_idx, double *topk_gate, double *load, double *prob_sum,
                    float *near_tie);

/* y[T][d] from expert rows Y[*][d] (row_of[T][k], -1 = dropped). */
void orc_combine(int T, int k, int d, const double *Y, const double *gate,
                 const int32_t *row_of, const float *x, int passthrough, double *y);

/* importance [n] and losses [8] from routing, counts, load, prob_sum. */
void orc_balance(int n, int T, int k, const int32_t *topk_idx, const double *topk_gate,
                 const int32_t *counts, const double *load, const double *prob_sum,
                 int64_t C, int router, double w_importance, double w_load, double alpha,
                 double *importance, double *losses);

/* Router statistics of the flat (or primary) gate, [MoE-intro] 第三部分:
 * *zsum = sum over tokens of the squared L2 norm of the clean logits
 * h = x W_g + b_g ("Router Z-loss" penalises the L2 norm of the logits before
 * the softmax); *hsum = sum over tokens of the entropy of softmax(h) over all
 * experts (the "gate entropy loss" rewards a high entropy).  0 or -1. */
int orc_router_stats(const orc_cfg *cfg, const orc_inputs *in, double *zsum, double *hsum);

/* Returns 0 on success, -1 on an invalid configuration.  losses [10]: [0..7]
 * as orc_balance; with router_stats, [8] = zsum / T and [9] = hsum / T of
 * orc_router_stats (else 0). */
int orc_forward(const orc_cfg *cfg, const orc_inputs *in, orc_outputs *out);

/* ---- backward pass ------------------------------------------------------ */
/* Gradients of
 *   L = sum_t <dy_t, y_t> + losses[0] + losses[1] + losses[3]
 *       + w_z * losses[8] - w_entropy * losses[9]
 * (an upstream gradient dy[T][d] of the layer output plus the weighted
 * balancing losses of orc_forward) with respect to x and every parameter.
 * For a hierarchical layer dWg, dbg, dWn are the primary gate's ([d][a],
 * [a], [d][a]), dWg2, dbg2, dWn2 the secondary gates' ([a][d][b], [a][b],
 * [a][d][b]), and dlogits / dnoise are not written.  With expert_bf16 the
 * rounding points of a mixed-precision backward are taken (see
 * orc_backward).  Any pointer other than dx and the routed experts' may be
 * NULL (not written). */
typedef struct {
  double *dx;                                 /* [T][d]                      */
  double *dWg, *dbg, *dWn;                    /* [d][n], [n], [d][n] (noise) */
  double *dW1, *db1, *dW2, *db2;              /* [n][f][d], [n][f], [n][d][f], [n][d] */
  double *dW1s, *db1s, *dW2s, *db2s;          /* shared expert: [f][d], [f], [d][f], [d] */
  double *dgate;                              /* [T][k] dL / d topk_gate      */
  double *dlogits;                            /* [T][n] dL / d (x W_g + b_g)  */
  double *dnoise;                             /* [T][n] dL / d (x W_noise)    */
  double *dWg2, *dbg2, *dWn2;                 /* hierarchical: [a][d][b], [a][b], [a][d][b] */
} orc_grads;

/* d CV(v)^2 / d v_i of orc_cv2 (0 where the mean is 0). */
void orc_cv2_grad(const double *v, int n, double *g);

/* 0, or -1 for a configuration the backward does not cover. */
int orc_backward(const orc_cfg *cfg, const orc_inputs *in, const float *dy, orc_grads *g);

/* One expert's part of the backward over nrows rows (the steps orc_backward
 * takes for each kept slot): row r is a token's input x_rows[r][d], the gate
 * g[r] of this expert in that token's output and the upstream gradient
 * dy_rows[r][d].  Adds to dW1 [f][d], db1 [f], dW2 [d][f], db2 [d] (db1, db2
 * may be NULL) and writes dgate[r] = <dy_r, E(x_r)> and dx_rows[r][d], the
 * expert's part of the input gradient. */
void orc_expert_backward(int d, int f, int bf16, int nrows, const float *x_rows, const double *g,
                         const float *dy_rows, const void *W1, const float *b1, const void *W2,
                         const float *b2, double *dW1, double *db1, double *dW2, double *db2,
                         double *dgate, double *dx_rows);

#ifdef __cplusplus
}
#endif
#endif
