/*
 * moe_oracle.c -- plain single-threaded CPU oracle of the Sparsely-Gated MoE
 * layer's forward and backward passes.  TEST INFRASTRUCTURE ONLY (see moe_oracle.h): it is
 * loaded by tests, the smoke check and the bench's CPU-baseline leg, never by
 * the product path.  Loops are written in the order of the formulas they
 * follow; no blocking, fusion or reordering beyond that.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ======================================================================= */
/* Noise: StandardNormal() of the noisy gate.                               */
/* [SGMoE-xyz] "Noisy Top-K 門控" writes H(x)_i = (x W_g)_i +                */
/* StandardNormal() * Softplus((x W_noise)_i) without saying how the normal */
/* deviate is drawn.  Our reading: a counter-based stream, so that every    */
/* (seed, token, expert, gate) has one fixed deviate on any machine:        */
/*   key = (seed low 32 bits, seed high 32 bits)                            */
/*   ctr = (token, expert / 4, gate_id, 0)                                  */
/*   the four words feed four consecutive experts 4m .. 4m+3: words (0,1)   */
/*   give the cosine and sine branches of one Box-Muller transform for      */
/*   experts 4m and 4m+1, words (2,3) those of a second one for 4m+2, 4m+3. */
/* ======================================================================= */

/* Philox4x32-10 [Philox]: ten rounds of the 4x32 S-box.  Each round
 * multiplies words 0 and 2 by the two round multipliers, swaps the halves and
 * folds in the key; the key is bumped by the two Weyl constants between
 * rounds. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;  /* round multipliers */
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;  /* key bumps (Weyl)  */
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t p0 = (uint64_t)M0 * (uint64_t)x0;
    uint64_t p1 = (uint64_t)M1 * (uint64_t)x2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t y0 = hi1 ^ x1 ^ k0;
    uint32_t y1 = lo1;
    uint32_t y2 = hi0 ^ x3 ^ k1;
    uint32_t y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Box-Muller [Box-Muller]: from two uniforms, r = sqrt(-2 ln u1) and angle
 * 2 pi u2 give two independent standard normals r cos(2 pi u2) (branch 0) and
 * r sin(2 pi u2) (branch 1).  u1 = (top 24 bits of w0 + 1)/2^24 lies in (0,1]
 * so the logarithm is finite; u2 = (top 24 bits of w1)/2^24 lies in [0,1). */
double orc_box_muller(uint32_t w0, uint32_t w1, int branch)
{
  double u1 = ((double)(w0 >> 8) + 1.0) / 16777216.0;
  double u2 = (double)(w1 >> 8) / 16777216.0;
  const double two_pi = 6.283185307179586476925286766559;
  double r = sqrt(-2.0 * log(u1));
  return branch ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

double orc_noise(uint64_t seed, uint32_t token, uint32_t expert, uint32_t gate_id)
{
  uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
  uint32_t ctr[4] = {token, expert >> 2, gate_id, 0u};
  uint32_t w[4];
  orc_philox4x32_10(ctr, key, w);
  uint32_t q = expert & 3u;
  return orc_box_muller(w[2 * (q >> 1)], w[2 * (q >> 1) + 1], (int)(q & 1u));
}

/* ======================================================================= */
/* Closed-form helpers                                                     */
/* ======================================================================= */

/* Softplus(z) = log(1 + e^z), written in the overflow-free form. */
double orc_softplus(double z)
{
  double a = fabs(z);
  return (z > 0.0 ? z : 0.0) + log1p(exp(-a));
}

/* Phi: the standard Normal CDF used by the smoothed load estimator
 * ([SGMoE-xyz] "負載平衡損失"). */
double orc_phi(double z)
{
  return 0.5 * erfc(-z / sqrt(2.0));
}

/* Squared coefficient of variation: population variance over squared mean.
 * [SGMoE-xyz] "負載平衡損失" defines L = w * CV(.)^2 without fixing the
 * variance convention; our reading is the population variance.  A zero mean
 * gives 0. */
double orc_cv2(const double *v, int n)
{
  if (n <= 0) return 0.0;
  double sum = 0.0;
  for (int i = 0; i < n; ++i) sum += v[i];
  double mean = sum / (double)n;
  if (mean == 0.0) return 0.0;
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += (v[i] - mean) * (v[i] - mean);
  double var = ss / (double)n;
  return var / (mean * mean);
}

/* Round an fp32 value to the nearest bf16 (ties to even), returned as fp32. */
float orc_bf16_round(float v)
{
  uint32_t u;
  memcpy(&u, &v, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u) {
    u = (u | 0x00400000u) & 0xffff0000u; /* keep NaN a (quiet) NaN */
  } else {
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    u &= 0xffff0000u;
  }
  float r;
  memcpy(&r, &u, 4);
  return r;
}

static double bf16_bits_to_double(uint16_t b)
{
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Expert capacity, [MoE-deep] §3.2: C = tokens per batch / E * capacity
 * factor.  With k slots per token our reading counts T*k routed slots, and
 * rounds up.  No limit when the factor is not positive. */
int64_t orc_capacity(int T, int k, int n, double capacity_factor)
{
  if (capacity_factor <= 0.0) return INT64_MAX;
  return (int64_t)ceil((double)T * (double)k * capacity_factor / (double)n);
}

/* ======================================================================= */
/* Gate                                                                     */
/* ======================================================================= */

typedef struct { float h; int i; } keyed;

/* Order: larger H first; equal H -> lower index first (the pages do not say
 * how ties are broken; our reading is lower index). */
static int keyed_cmp(const void *pa, const void *pb)
{
  const keyed *a = (const keyed *)pa, *b = (const keyed *)pb;
  if (a->h > b->h) return -1;
  if (a->h < b->h) return 1;
  return (a->i < b->i) ? -1 : (a->i > b->i);
}

/* Noisy top-k gating, [SGMoE-xyz] "Noisy Top-K 門控" and [SGMoE-note] "Noisy
 * Top-K Gating":
 *   H(x)_i = (x W_g)_i + StandardNormal() * Softplus((x W_noise)_i)
 *   KeepTopK(v,k)_i = v_i if v_i is among the top k of v, else -inf
 *   G(x) = Softmax(KeepTopK(H(x), k))
 * The optional per-expert bias b_g is part of the clean logit (x W_g)_i.
 * Router 1 is the Switch router of [MoE-deep] §3.1: p = softmax(x W_r) over
 * all experts, the token goes to argmax p and is weighted by p_argmax (no
 * renormalisation over the kept expert). */
void orc_gate_row(int d, int n, int k, int router, int noise, uint64_t seed,
                  uint32_t token, uint32_t gate_id, const float *x,
                  const float *Wg, const float *bg, const float *Wn,
                  double *c, double *s, float *H, int *order, double *gates,
                  double *p, const float *sel_bias)
{
  for (int i = 0; i < n; ++i) { c[i] = 0.0; s[i] = 0.0; }
  for (int j = 0; j < d; ++j) {
    double xj = (double)x[j];
    for (int i = 0; i < n; ++i) c[i] += xj * (double)Wg[(size_t)j * n + i];
    if (noise)
      for (int i = 0; i < n; ++i) s[i] += xj * (double)Wn[(size_t)j * n + i];
  }
  for (int i = 0; i < n; ++i) {
    if (bg) c[i] += (double)bg[i];
    if (noise) {
      s[i] = orc_softplus(s[i]);
      double eps = orc_noise(seed, token, (uint32_t)i, gate_id);
      H[i] = (float)(c[i] + eps * s[i]);
    } else {
      s[i] = 0.0;
      /* router 2 ranks the routing score c + b ([MoE-deep] §6.3: the bias
       * enters the selection only) */
      H[i] = (float)(router == 2 && sel_bias ? c[i] + (double)sel_bias[i] : c[i]);
    }
  }

  keyed *kv = (keyed *)malloc(sizeof(keyed) * (size_t)n);
  for (int i = 0; i < n; ++i) { kv[i].h = H[i]; kv[i].i = i; }
  qsort(kv, (size_t)n, sizeof(keyed), keyed_cmp);
  for (int i = 0; i < n; ++i) order[i] = kv[i].i;
  free(kv);

  if (router == 1) {
    double m = c[0];
    for (int i = 1; i < n; ++i) if (c[i] > m) m = c[i];
    double den = 0.0;
    for (int i = 0; i < n; ++i) den += exp(c[i] - m);
    for (int i = 0; i < n; ++i) {
      double pi = exp(c[i] - m) / den;
      if (p) p[i] = pi;
      if (i == order[0]) gates[0] = pi;
    }
    return;
  }

  if (router == 2) {
    /* [MoE-deep] §6.2: s_i = Sigmoid(h_i) of the logits without the bias,
     * g_i = s_i / sum of s_j over the kept k */
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += 1.0 / (1.0 + exp(-c[order[j]]));
    for (int j = 0; j < k; ++j) gates[j] = (1.0 / (1.0 + exp(-c[order[j]]))) / den;
    return;
  }

  /* softmax over the kept k; every other entry is -inf and gets 0. */
  double hmax = (double)H[order[0]];
  double den = 0.0;
  for (int j = 0; j < k; ++j) den += exp((double)H[order[j]] - hmax);
  for (int j = 0; j < k; ++j) gates[j] = exp((double)H[order[j]] - hmax) / den;
}

/* Smoothed load, [SGMoE-xyz] "負載平衡損失":
 *   P(x,i) = Phi( ((x W_g)_i - kth_excluding(H(x), k, i)) / Softplus((x W_noise)_i) )
 * kth_excluding(H,k,i) is the k-th largest entry of H once entry i is left
 * out.  With H sorted, that is the (k+1)-th largest when i itself is among the
 * first k, and the k-th largest otherwise; -inf (P = 1) when fewer than k
 * other entries exist.  Without noise the estimator has no spread; we use
 * its zero-noise limit, the indicator of i being kept. */
void orc_load_row(int n, int k, int noise, const double *c, const double *s,
                  const float *H, double *P)
{
  int *rank = (int *)malloc(sizeof(int) * (size_t)n);
  keyed *kv = (keyed *)malloc(sizeof(keyed) * (size_t)n);
  for (int i = 0; i < n; ++i) { kv[i].h = H[i]; kv[i].i = i; }
  qsort(kv, (size_t)n, sizeof(keyed), keyed_cmp);
  for (int r = 0; r < n; ++r) rank[kv[r].i] = r;
  double v_k = (double)kv[k - 1].h;
  double v_k1 = (k < n) ? (double)kv[k].h : -INFINITY;
  for (int i = 0; i < n; ++i) {
    int kept = rank[i] < k;
    if (!noise) { P[i] = kept ? 1.0 : 0.0; continue; }
    double thr = kept ? v_k1 : v_k;
    if (thr == -INFINITY) { P[i] = 1.0; continue; }
    double num = c[i] - thr;
    if (s[i] == 0.0) { P[i] = num > 0.0 ? 1.0 : (num < 0.0 ? 0.0 : 0.5); continue; }
    P[i] = orc_phi(num / s[i]);
  }
  free(kv);
  free(rank);
}

/* ======================================================================= */
/* Dispatch                                                                 */
/* ======================================================================= */

/* [SGMoE-note] "Sparsely-Gated MoE 层架构": E_i(x) need not be computed when
 * G(x)_i = 0, so each token is sent only to its kept experts.  Slots are
 * visited token by token, slot by slot; a slot's rank is the number of
 * earlier slots sent to the same expert.  [MoE-deep] §3.2: an expert takes
 * at most C tokens, the rest overflow (our reading: the later tokens, in
 * this visiting order, are the ones that overflow). */
void orc_dispatch(int T, int k, int n, int64_t C, const int32_t *idx,
                  int32_t *counts, int32_t *offsets, int32_t *perm_token,
                  int32_t *perm_slot, int32_t *row_of, int64_t *n_invalid)
{
  int64_t invalid = 0;
  for (int e = 0; e < n; ++e) counts[e] = 0;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int32_t e = idx[(size_t)t * k + j];
      if (e < 0 || e >= n) invalid++;
      else counts[e]++;
    }
  offsets[0] = 0;
  for (int e = 0; e < n; ++e) {
    int64_t kept = counts[e] < C ? counts[e] : C;
    offsets[e + 1] = offsets[e] + (int32_t)kept;
  }
  int32_t *seen = (int32_t *)calloc((size_t)(n > 0 ? n : 1), sizeof(int32_t));
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      size_t p = (size_t)t * k + j;
      int32_t e = idx[p];
      if (e < 0 || e >= n) { row_of[p] = -1; continue; }
      int32_t r = seen[e]++;
      if ((int64_t)r < C) {
        int32_t row = offsets[e] + r;
        row_of[p] = row;
        perm_token[row] = t;
        perm_slot[row] = j;
      } else {
        row_of[p] = -1;
      }
    }
  free(seen);
  if (n_invalid) *n_invalid = invalid;
}

/* ======================================================================= */
/* Expert                                                                   */
/* ======================================================================= */

/* [SGMoE-note] "Sparsely-Gated MoE 层架构": every expert is a feed-forward
 * network with one ReLU hidden layer, same shape, own parameters:
 *   E(x) = ReLU(x W1^T + b1) W2^T + b2      (W1: [f][d], W2: [d][f])
 * bf16 experts take bf16 activations: x and the hidden layer are rounded to
 * bf16, all sums are fp64. */
void orc_expert_row(int d, int f, int bf16, const float *x, const void *W1,
                    const float *b1, const void *W2, const float *b2, double *y)
{
  double *h = (double *)malloc(sizeof(double) * (size_t)(f > 0 ? f : 1));
  for (int j = 0; j < f; ++j) {
    double acc = 0.0;
    for (int q = 0; q < d; ++q) {
      double xv, wv;
      if (bf16) {
        xv = (double)orc_bf16_round(x[q]);
        wv = bf16_bits_to_double(((const uint16_t *)W1)[(size_t)j * d + q]);
      } else {
        xv = (double)x[q];
        wv = (double)((const float *)W1)[(size_t)j * d + q];
      }
      acc += xv * wv;
    }
    if (b1) acc += (double)b1[j];
    double r = acc > 0.0 ? acc : 0.0;
    h[j] = bf16 ? (double)orc_bf16_round((float)r) : r;
  }
  for (int q = 0; q < d; ++q) {
    double acc = 0.0;
    for (int j = 0; j < f; ++j) {
      double wv = bf16 ? bf16_bits_to_double(((const uint16_t *)W2)[(size_t)q * f + j])
                       : (double)((const float *)W2)[(size_t)q * f + j];
      acc += h[j] * wv;
    }
    if (b2) acc += (double)b2[q];
    y[q] = acc;
  }
  free(h);
}

/* ======================================================================= */
/* Whole layer                                                              */
/* ======================================================================= */

static float min_gap(const float *H, const int *order, int n, int k)
{
  float g = INFINITY;
  int last = k < n - 1 ? k : n - 1;
  for (int j = 1; j <= last; ++j) {
    float d = H[order[j - 1]] - H[order[j]];
    if (d < g) g = d;
  }
  return g;
}

static int valid_cfg(const orc_cfg *c)
{
  if (c->T < 0 || c->d < 1 || c->f < 1 || c->n < 1 || c->k < 1 || c->k > c->n) return 0;
  if (c->router != 0 && c->router != 1 && c->router != 2) return 0;
  if (c->router == 1 && (c->k != 1 || c->noise || c->hier_a)) return 0;
  if (c->router == 2 && (c->noise || c->hier_a)) return 0;
  if (c->hier_a) {
    if (c->hier_b < 1 || c->hier_a * c->hier_b != c->n) return 0;
    if (c->hier_k1 < 1 || c->hier_k1 > c->hier_a) return 0;
    if (c->hier_k2 < 1 || c->hier_k2 > c->hier_b) return 0;
    if (c->hier_k1 * c->hier_k2 != c->k) return 0;
  }
  return 1;
}

int orc_gate_tokens(const orc_cfg *cfg, const orc_inputs *in, const int32_t *tokens, int ntok,
                    int32_t *topk_idx, double *topk_gate, double *load, double *prob_sum,
                    float *near_tie);

/* Gate over a whole batch (flat, Switch or hierarchical): topk_idx /
 * topk_gate [T][k], load [n] (smoothed load, or its zero-noise limit),
 * prob_sum [n] (Switch: sum of router probabilities; else 0), near_tie [T]
 * (smallest gap between neighbouring sorted logits among the first k+1 of any
 * gate that decided the token; may be NULL).
 *
 * Hierarchical layer ([SGMoE-note] "分层 MoE"): the primary gate picks k1
 * groups, group i's own gate picks k2 of its b experts for the tokens sent
 * to it; expert (i,j) has flat id i*b+j and gate G_p(x)_i * G_i(x)_j; slot
 * order is primary slot major.  Load (our reading, parity unpinned beyond
 * the zero-noise limit): Load(i*b+j) = Load_p(X)_i * Load_i(X_i)_j / |X_i|. */
int orc_gate_batch(const orc_cfg *cfg, const orc_inputs *in, int32_t *topk_idx,
                   double *topk_gate, double *load, double *prob_sum, float *near_tie)
{
  return orc_gate_tokens(cfg, in, NULL, cfg->T, topk_idx, topk_gate, load, prob_sum, near_tie);
}

/* The gate for a list of tokens (row r of the outputs is token tokens[r]:
 * its x row and its noise counter); tokens == NULL means 0 .. ntok-1.  load
 * and prob_sum are summed over the listed tokens only (for the hierarchical
 * layer Load is a whole-batch quantity and is only meaningful for the whole
 * batch). */
int orc_gate_tokens(const orc_cfg *cfg, const orc_inputs *in, const int32_t *tokens, int ntok,
                    int32_t *topk_idx, double *topk_gate, double *load, double *prob_sum,
                    float *near_tie)
{
  if (!valid_cfg(cfg)) return -1;
  const int T = ntok, d = cfg->d, n = cfg->n, k = cfg->k;
  const int hier = cfg->hier_a > 0;
  const int ng = hier ? (cfg->hier_a > cfg->hier_b ? cfg->hier_a : cfg->hier_b) : n;

  double *c = (double *)malloc(sizeof(double) * (size_t)ng);
  double *s = (double *)malloc(sizeof(double) * (size_t)ng);
  double *P = (double *)malloc(sizeof(double) * (size_t)ng);
  double *pr = (double *)malloc(sizeof(double) * (size_t)ng);
  float *H = (float *)malloc(sizeof(float) * (size_t)ng);
  int *order = (int *)malloc(sizeof(int) * (size_t)ng);
  double *g1 = (double *)malloc(sizeof(double) * (size_t)(k + 1));
  double *g2 = (double *)malloc(sizeof(double) * (size_t)(k + 1));
  int *pidx = (int *)malloc(sizeof(int) * (size_t)(k + 1));

  for (int e = 0; e < n; ++e) {
    load[e] = 0.0;
    if (prob_sum) prob_sum[e] = 0.0;
  }

  if (!hier) {
    for (int t = 0; t < T; ++t) {
      const int tok = tokens ? tokens[t] : t;
      const float *xt = in->x + (size_t)tok * d;
      orc_gate_row(d, n, k, cfg->router, cfg->noise, cfg->seed, (uint32_t)tok, 0u,
                   xt, in->Wg, in->bg, in->Wn, c, s, H, order, g1, pr, in->sel_bias);
      for (int j = 0; j < k; ++j) {
        topk_idx[(size_t)t * k + j] = order[j];
        topk_gate[(size_t)t * k + j] = g1[j];
      }
      orc_load_row(n, k, cfg->noise, c, s, H, P);
      for (int i = 0; i < n; ++i) load[i] += P[i];
      if (cfg->router == 1 && prob_sum)
        for (int i = 0; i < n; ++i) prob_sum[i] += pr[i];
      if (near_tie) near_tie[t] = min_gap(H, order, n, k);
    }
  } else {
    const int a = cfg->hier_a, b = cfg->hier_b, k1 = cfg->hier_k1, k2 = cfg->hier_k2;
    double *load_p = (double *)calloc((size_t)a, sizeof(double));
    double *load_s = (double *)calloc((size_t)a * b, sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)a, sizeof(int64_t));
    for (int t = 0; t < T; ++t) {
      const int tok = tokens ? tokens[t] : t;
      const float *xt = in->x + (size_t)tok * d;
      orc_gate_row(d, a, k1, 0, cfg->noise, cfg->seed, (uint32_t)tok, 0u, xt,
                   in->Wg, in->bg, in->Wn, c, s, H, order, g1, NULL, NULL);
      float gap = min_gap(H, order, a, k1);
      orc_load_row(a, k1, cfg->noise, c, s, H, P);
      for (int i = 0; i < a; ++i) load_p[i] += P[i];
      for (int ps = 0; ps < k1; ++ps) pidx[ps] = order[ps];
      for (int ps = 0; ps < k1; ++ps) {
        int gi = pidx[ps];
        cnt[gi]++;
        const float *Wg2 = in->Wg2 + (size_t)gi * d * b;
        const float *Wn2 = in->Wn2 ? in->Wn2 + (size_t)gi * d * b : NULL;
        const float *bg2 = in->bg2 ? in->bg2 + (size_t)gi * b : NULL;
        orc_gate_row(d, b, k2, 0, cfg->noise, cfg->seed, (uint32_t)tok, (uint32_t)(1 + gi),
                     xt, Wg2, bg2, Wn2, c, s, H, order, g2, NULL, NULL);
        float gap2 = min_gap(H, order, b, k2);
        if (gap2 < gap) gap = gap2;
        orc_load_row(b, k2, cfg->noise, c, s, H, P);
        for (int j = 0; j < b; ++j) load_s[(size_t)gi * b + j] += P[j];
        for (int ss = 0; ss < k2; ++ss) {
          size_t slot = (size_t)t * k + (size_t)ps * k2 + ss;
          topk_idx[slot] = gi * b + order[ss];
          topk_gate[slot] = g1[ps] * g2[ss];
        }
      }
      if (near_tie) near_tie[t] = gap;
    }
    for (int i = 0; i < a; ++i)
      for (int j = 0; j < b; ++j)
        load[(size_t)i * b + j] =
            cnt[i] > 0 ? load_p[i] * load_s[(size_t)i * b + j] / (double)cnt[i] : 0.0;
    free(load_p); free(load_s); free(cnt);
  }
  free(c); free(s); free(P); free(pr); free(H); free(order); free(g1); free(g2); free(pidx);
  return 0;
}

/* Gate-weighted sum of expert rows, y = sum_i G(x)_i E_i(x) ([SGMoE-note]
 * "Sparsely-Gated MoE 层架构"), with E_i(x) already computed as row
 * row_of[t][j] of Y.  A dropped slot (row -1) adds nothing and the other
 * gates are not renormalised (the pages are silent; plainest reading).  A
 * token whose every slot was dropped passes through the residual ([MoE-deep]
 * §3.2): with passthrough its output is x, else 0. */
void orc_combine(int T, int k, int d, const double *Y, const double *gate,
                 const int32_t *row_of, const float *x, int passthrough, double *y)
{
  for (int t = 0; t < T; ++t) {
    double *yt = y + (size_t)t * d;
    for (int q = 0; q < d; ++q) yt[q] = 0.0;
    int kept = 0;
    for (int j = 0; j < k; ++j) {
      int32_t r = row_of[(size_t)t * k + j];
      if (r < 0) continue;
      kept++;
      double g = gate[(size_t)t * k + j];
      for (int q = 0; q < d; ++q) yt[q] += g * Y[(size_t)r * d + q];
    }
    if (kept == 0 && passthrough)
      for (int q = 0; q < d; ++q) yt[q] = (double)x[(size_t)t * d + q];
  }
}

/* Balancing statistics ([SGMoE-xyz] "負載平衡損失"; [MoE-deep] §3.2):
 * importance[i] = sum over tokens of G(x)_i (from the kept-expert lists);
 * losses[0] L_importance = w_importance * CV(Importance)^2
 * losses[1] L_load       = w_load * CV(Load)^2
 * losses[2] N * sum_i f_i P_i  (Switch; f_i = counts_i / T, before the
 *           capacity cut, P_i = prob_sum_i / T), 0 for router 0
 * losses[3] alpha * losses[2]
 * losses[4] dropped slots / (T k)  (dropped = sum_i max(counts_i - C, 0))
 * losses[5] CV(Importance)^2, losses[6] CV(Load)^2, losses[7] dropped slots */
void orc_balance(int n, int T, int k, const int32_t *topk_idx, const double *topk_gate,
                 const int32_t *counts, const double *load, const double *prob_sum,
                 int64_t C, int router, double w_importance, double w_load, double alpha,
                 double *importance, double *losses)
{
  for (int e = 0; e < n; ++e) importance[e] = 0.0;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int32_t e = topk_idx[(size_t)t * k + j];
      if (e >= 0 && e < n) importance[e] += topk_gate[(size_t)t * k + j];
    }
  double dropped = 0.0;
  for (int e = 0; e < n; ++e)
    if ((int64_t)counts[e] > C) dropped += (double)((int64_t)counts[e] - C);
  double aux = 0.0;
  if (router == 1 && T > 0 && prob_sum) {
    for (int i = 0; i < n; ++i)
      aux += ((double)counts[i] / (double)T) * (prob_sum[i] / (double)T);
    aux *= (double)n;
  }
  double cv2_imp = orc_cv2(importance, n);
  double cv2_load = orc_cv2(load, n);
  double S = (double)T * (double)k;
  losses[0] = w_importance * cv2_imp;
  losses[1] = w_load * cv2_load;
  losses[2] = aux;
  losses[3] = alpha * aux;
  losses[4] = S > 0 ? dropped / S : 0.0;
  losses[5] = cv2_imp;
  losses[6] = cv2_load;
  losses[7] = dropped;
}

/* The whole layer, y = sum_i G(x)_i E_i(x) over the kept experts
 * ([SGMoE-note] "Sparsely-Gated MoE 层架构"): gate, capacity-limited
 * dispatch, each kept expert applied to the token directly, gate-weighted
 * sum, pass-through of fully dropped tokens, balancing statistics.  Losses
 * as in orc_balance. */
/* [MoE-deep] §6.3: the bias of an overloaded expert goes down by gamma, that
 * of an underloaded one up by gamma.  Our reading of over / under: more / fewer
 * slots than the average T*k/n (compared exactly: counts*n against T*k); an
 * expert exactly at the average keeps its bias. */
void orc_sel_bias_update(int n, int T, int k, const int32_t *counts, float gamma, float *bias)
{
  const int64_t total = (int64_t)T * k;
  for (int i = 0; i < n; ++i) {
    const int64_t scaled = (int64_t)counts[i] * n;
    if (scaled > total) bias[i] = bias[i] - gamma;
    else if (scaled < total) bias[i] = bias[i] + gamma;
  }
}

int orc_router_stats(const orc_cfg *cfg, const orc_inputs *in, double *zsum, double *hsum)
{
  if (!valid_cfg(cfg)) return -1;
  const int d = cfg->d, ng = cfg->hier_a > 0 ? cfg->hier_a : cfg->n;
  double *c = (double *)malloc(sizeof(double) * (size_t)ng);
  double z = 0.0, h = 0.0;
  for (int t = 0; t < cfg->T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    for (int i = 0; i < ng; ++i) c[i] = in->bg ? (double)in->bg[i] : 0.0;
    for (int j = 0; j < d; ++j)
      for (int i = 0; i < ng; ++i) c[i] += (double)xt[j] * (double)in->Wg[(size_t)j * ng + i];
    double m = c[0];
    for (int i = 0; i < ng; ++i) {
      z += c[i] * c[i];
      if (c[i] > m) m = c[i];
    }
    /* entropy of p = softmax(c): -sum p_i log p_i with log p_i = c_i - m - log S */
    double S = 0.0;
    for (int i = 0; i < ng; ++i) S += exp(c[i] - m);
    double ent = 0.0;
    for (int i = 0; i < ng; ++i) {
      double p = exp(c[i] - m) / S;
      if (p > 0.0) ent -= p * (c[i] - m - log(S));
    }
    h += ent;
  }
  free(c);
  *zsum = z;
  *hsum = h;
  return 0;
}

int orc_forward(const orc_cfg *cfg, const orc_inputs *in, orc_outputs *out)
{
  if (cfg->shared_expert && (!in->W1s || !in->W2s)) return -1;
  if (orc_gate_batch(cfg, in, out->topk_idx, out->topk_gate, out->load, out->prob_sum,
                     out->near_tie) != 0)
    return -1;
  const int T = cfg->T, d = cfg->d, n = cfg->n, k = cfg->k, f = cfg->f;
  int64_t C = orc_capacity(T, k, n, cfg->capacity_factor);
  int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
  size_t S = (size_t)T * k;
  int32_t *perm_token = (int32_t *)malloc(sizeof(int32_t) * (S > 0 ? S : 1));
  int32_t *perm_slot = (int32_t *)malloc(sizeof(int32_t) * (S > 0 ? S : 1));
  orc_dispatch(T, k, n, C, out->topk_idx, out->counts, offsets, perm_token, perm_slot,
               out->row_of, NULL);

  double *ye = (double *)malloc(sizeof(double) * (size_t)d);
  const size_t w1_stride = (size_t)f * d, w2_stride = (size_t)d * f;
  const size_t esz = cfg->expert_bf16 ? 2 : 4;
  for (int t = 0; t < T; ++t) {
    double *yt = out->y + (size_t)t * d;
    for (int q = 0; q < d; ++q) yt[q] = 0.0;
    int kept_slots = 0;
    for (int j = 0; j < k; ++j) {
      size_t pj = (size_t)t * k + j;
      if (out->row_of[pj] < 0) continue;
      kept_slots++;
      int e = out->topk_idx[pj];
      const char *W1e = (const char *)in->W1 + (size_t)e * w1_stride * esz;
      const char *W2e = (const char *)in->W2 + (size_t)e * w2_stride * esz;
      const float *b1e = in->b1 ? in->b1 + (size_t)e * f : NULL;
      const float *b2e = in->b2 ? in->b2 + (size_t)e * d : NULL;
      orc_expert_row(d, f, cfg->expert_bf16, in->x + (size_t)t * d, W1e, b1e, W2e, b2e, ye);
      double g = out->topk_gate[pj];
      for (int q = 0; q < d; ++q) yt[q] += g * ye[q];
    }
    if (kept_slots == 0 && k > 0 && cfg->passthrough)
      for (int q = 0; q < d; ++q) yt[q] = (double)in->x[(size_t)t * d + q];
    if (cfg->shared_expert) {
      /* [MoE-deep] §5.2 / §6.2: y = E_shared(x) + sum_j g_j E_j(x); one
       * shared expert with weight 1 (DeepSeek-V3's form).  Our reading: a
       * token whose routed slots all overflowed keeps its shared-expert term
       * (the pass-through replaces only the routed sum). */
      orc_expert_row(d, f, cfg->expert_bf16, in->x + (size_t)t * d, in->W1s, in->b1s, in->W2s,
                     in->b2s, ye);
      for (int q = 0; q < d; ++q) yt[q] += ye[q];
    }
  }

  orc_balance(n, T, k, out->topk_idx, out->topk_gate, out->counts, out->load, out->prob_sum, C,
              cfg->router, cfg->w_importance, cfg->w_load, cfg->alpha, out->importance,
              out->losses);
  out->losses[8] = out->losses[9] = 0.0;
  if (cfg->router_stats && T > 0) {
    double zs, hs;
    orc_router_stats(cfg, in, &zs, &hs);
    out->losses[8] = zs / T;
    out->losses[9] = hs / T;
  }
  free(ye); free(offsets); free(perm_token); free(perm_slot);
  return 0;
}

/* ======================================================================= */
/* Backward pass                                                            */
/* ======================================================================= */
/*
 * The pages give no backward formulas; they say which paths carry a
 * gradient.  The kept gates are a smooth function of the logits, so the
 * gradient reaches the gate network through them ([SGMoE-xyz] 常見問題);
 * KeepTopK gives the experts it drops none ([SGMoE-note] 缺点与局限性); the
 * noise lets the load loss reach the gate through Phi ([SGMoE-note] Noisy
 * Top-K Gating).  orc_backward is the chain rule of orc_forward, taken in the
 * reverse order of its steps: combine, experts, dispatch, gate.
 *
 * Mixed precision (expert_bf16): the kernels keep every expert-side
 * activation gradient in bf16 and accumulate in fp32, so the oracle rounds
 * where they store: the gradient reaching an expert row, g * dy (the product
 * taken in fp32, as g is an fp32 output of the gate); the hidden-layer
 * gradient after the ReLU mask; the input-row gradient of each expert.  The
 * combine's gate gradient uses the expert output rounded to bf16, the value
 * the combine summed.  Everything else is fp64.
 */

void orc_cv2_grad(const double *v, int n, double *g)
{
  /* CV^2 = var / mean^2 with var = sum (v_i - mean)^2 / n:
   * d var / d v_i = 2 (v_i - mean) / n, d mean / d v_i = 1 / n, so
   * d CV^2 / d v_i = 2 / (n mean^2) * ((v_i - mean) - var / mean). */
  double sum = 0.0;
  for (int i = 0; i < n; ++i) sum += v[i];
  double mean = n > 0 ? sum / (double)n : 0.0;
  if (mean == 0.0) {
    for (int i = 0; i < n; ++i) g[i] = 0.0;
    return;
  }
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += (v[i] - mean) * (v[i] - mean);
  double var = ss / (double)n;
  for (int i = 0; i < n; ++i)
    g[i] = 2.0 / ((double)n * mean * mean) * ((v[i] - mean) - var / mean);
}

static double wval(const void *W, int bf16, size_t i)
{
  return bf16 ? bf16_bits_to_double(((const uint16_t *)W)[i]) : (double)((const float *)W)[i];
}

static double rnd(int bf16, double v)
{
  return bf16 ? (double)orc_bf16_round((float)v) : v;
}

/* One expert on one row, forward and backward.  dyr: the gradient reaching
 * the layer output row; gate: the weight of this expert's output in it (1 for
 * the shared expert).  Adds to dW1 [f][d], db1 [f], dW2 [d][f], db2 [d] and
 * dxr [d]; returns <dyr, E(x)> (the gradient of the gate). */
static double expert_row_bwd(int d, int f, int bf16, const float *x, const void *W1,
                             const float *b1, const void *W2, const float *b2, double gate,
                             const float *dyr, double *dW1, double *db1, double *dW2, double *db2,
                             double *dxr)
{
  double *xv = (double *)malloc(sizeof(double) * (size_t)d);
  double *h = (double *)malloc(sizeof(double) * (size_t)f);
  double *dh = (double *)malloc(sizeof(double) * (size_t)f);
  double *dyp = (double *)malloc(sizeof(double) * (size_t)d);
  for (int q = 0; q < d; ++q) xv[q] = rnd(bf16, (double)x[q]);
  /* forward: h = ReLU(W1 x + b1), E = W2 h + b2 */
  for (int j = 0; j < f; ++j) {
    double a = b1 ? (double)b1[j] : 0.0;
    for (int q = 0; q < d; ++q) a += wval(W1, bf16, (size_t)j * d + q) * xv[q];
    h[j] = rnd(bf16, a > 0.0 ? a : 0.0);
  }
  double dgate = 0.0;
  for (int q = 0; q < d; ++q) {
    double e = b2 ? (double)b2[q] : 0.0;
    for (int j = 0; j < f; ++j) e += wval(W2, bf16, (size_t)q * f + j) * h[j];
    dgate += (double)dyr[q] * rnd(bf16, e);
  }
  /* dE = gate * dy */
  for (int q = 0; q < d; ++q)
    dyp[q] = bf16 ? (double)orc_bf16_round((float)gate * dyr[q]) : gate * (double)dyr[q];
  /* E = W2 h + b2: dW2 += dE h^T, db2 += dE, dh = W2^T dE */
  for (int q = 0; q < d; ++q) {
    if (db2) db2[q] += dyp[q];
    for (int j = 0; j < f; ++j) dW2[(size_t)q * f + j] += dyp[q] * h[j];
  }
  for (int j = 0; j < f; ++j) {
    double acc = 0.0;
    for (int q = 0; q < d; ++q) acc += wval(W2, bf16, (size_t)q * f + j) * dyp[q];
    /* ReLU passes the gradient where its output is positive */
    dh[j] = rnd(bf16, h[j] > 0.0 ? acc : 0.0);
  }
  /* a = W1 x + b1: dW1 += dh x^T, db1 += dh, dx = W1^T dh */
  for (int j = 0; j < f; ++j) {
    if (db1) db1[j] += dh[j];
    for (int q = 0; q < d; ++q) dW1[(size_t)j * d + q] += dh[j] * xv[q];
  }
  for (int q = 0; q < d; ++q) {
    double acc = 0.0;
    for (int j = 0; j < f; ++j) acc += wval(W1, bf16, (size_t)j * d + q) * dh[j];
    dxr[q] += rnd(bf16, acc);
  }
  free(xv); free(h); free(dh); free(dyp);
  return dgate;
}

void orc_expert_backward(int d, int f, int bf16, int nrows, const float *x_rows, const double *g,
                         const float *dy_rows, const void *W1, const float *b1, const void *W2,
                         const float *b2, double *dW1, double *db1, double *dW2, double *db2,
                         double *dgate, double *dx_rows)
{
  for (int r = 0; r < nrows; ++r) {
    double *dxr = dx_rows + (size_t)r * d;
    for (int q = 0; q < d; ++q) dxr[q] = 0.0;
    dgate[r] = expert_row_bwd(d, f, bf16, x_rows + (size_t)r * d, W1, b1, W2, b2, g[r],
                              dy_rows + (size_t)r * d, dW1, db1, dW2, db2, dxr);
  }
}

/* One noisy top-k softmax level of a gate ([SGMoE-xyz] "Noisy Top-K 門控"),
 * backward: H = c + eps s, G = Softmax over the kept k of H, s = Softplus(z),
 * z = x W_noise.  In: the row's c, s, H and order (orc_gate_row), its kept
 * gates gk and dL/dG of them (dG), the load-loss coefficient of each column
 * (lam_load, NULL without a load term), the noise stream's (token, gate id).
 * Out: dc [m] (dL/dc) and dz [m] (dL/dz, noise only); scratch dH [m], rank [m].
 * The load term differentiates P(x,i) = Phi((c_i - thr_i) / s_i) in c_i, s_i
 * and in the H of the expert that fixes thr_i, as in orc_backward. */
static void level_bwd(int m, int k, int noise, uint64_t seed, uint32_t tok, uint32_t gate_id,
                      const float *xt, int d, const float *Wn, const double *c, const double *s,
                      const float *H, const int *order, const double *gk, const double *dG,
                      const double *lam_load, double *dc, double *dz, double *dH, int *rank)
{
  for (int r = 0; r < m; ++r) rank[order[r]] = r;
  for (int i = 0; i < m; ++i) dc[i] = dz[i] = dH[i] = 0.0;
  double sum = 0.0;
  for (int j = 0; j < k; ++j) sum += gk[j] * dG[j];
  for (int j = 0; j < k; ++j) dH[order[j]] = gk[j] * (dG[j] - sum);
  if (noise && lam_load) {
    const int jk = order[k - 1], jk1 = k < m ? order[k] : -1;
    for (int i = 0; i < m; ++i) {
      const int jt = rank[i] < k ? jk1 : jk;
      if (jt < 0 || s[i] == 0.0) continue;
      const double u = (c[i] - (double)H[jt]) / s[i];
      const double a = lam_load[i] * exp(-0.5 * u * u) / sqrt(2.0 * acos(-1.0)) / s[i];
      dc[i] += a;
      dz[i] -= a * u;
      dH[jt] -= a;
    }
  }
  for (int i = 0; i < m; ++i) {
    dc[i] += dH[i];
    if (noise) dz[i] += dH[i] * orc_noise(seed, tok, (uint32_t)i, gate_id);
  }
  if (noise)
    for (int i = 0; i < m; ++i) {
      double z = 0.0;
      for (int q = 0; q < d; ++q) z += (double)xt[q] * (double)Wn[(size_t)q * m + i];
      dz[i] *= 1.0 / (1.0 + exp(-z));
    }
}

/* The backward of a gate level's projections c = x W + bias, z = x W_noise
 * (W, W_noise [d][m]): adds x dc^T to dW, dc to db, x dz^T to dWn and
 * W dc + W_noise dz to dxt. */
static void level_proj_bwd(int d, int m, int noise, const float *xt, const float *W, const float *Wn,
                           const double *dc, const double *dz, double *dW, double *db, double *dWn,
                           double *dxt)
{
  for (int q = 0; q < d; ++q) {
    double acc = 0.0;
    for (int i = 0; i < m; ++i) {
      acc += W[(size_t)q * m + i] * dc[i];
      if (dW) dW[(size_t)q * m + i] += (double)xt[q] * dc[i];
      if (noise) {
        acc += Wn[(size_t)q * m + i] * dz[i];
        if (dWn) dWn[(size_t)q * m + i] += (double)xt[q] * dz[i];
      }
    }
    dxt[q] += acc;
  }
  if (db)
    for (int i = 0; i < m; ++i) db[i] += dc[i];
}

/* The hierarchical layer ([SGMoE-note] "分层 MoE"): token t's slot ps*k2+ss
 * is expert gi*b + j, gi the ps-th kept group of the primary gate and j the
 * ss-th kept expert of gi's gate, with gate G_p(x)_gi G_gi(x)_j.  Importance
 * sums the slot gates; Load(gi*b+j) = Load_p(X)_gi Load_gi(X_gi)_j / |X_gi|,
 * the forward's reading, |X_gi| a count (no gradient): so the load loss
 * reaches the primary level through lam_p(gi) = sum_j lamL(gi*b+j)
 * Load_gi_j / |X_gi| and group gi's level through lam_s(gi, j) =
 * lamL(gi*b+j) Load_p_gi / |X_gi|.  Each level's chain rule is that of the
 * flat gate (level_bwd); the experts and the combine are the flat layer's. */
static int orc_backward_hier(const orc_cfg *cfg, const orc_inputs *in, const float *dy, orc_grads *g)
{
  const int T = cfg->T, d = cfg->d, n = cfg->n, k = cfg->k, f = cfg->f, bf16 = cfg->expert_bf16;
  const int a = cfg->hier_a, b = cfg->hier_b, k1 = cfg->hier_k1, k2 = cfg->hier_k2;
  const int noise = cfg->noise;
  const size_t esz = bf16 ? 2 : 4;
  const size_t S = (size_t)T * k;
  const int mx = a > b ? a : b;

  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  double *gate = (double *)malloc(sizeof(double) * (S ? S : 1));
  double *load = (double *)malloc(sizeof(double) * (size_t)n);
  double *psum = (double *)malloc(sizeof(double) * (size_t)n);
  double *imp = (double *)calloc((size_t)n, sizeof(double));
  int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
  int32_t *ptok = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  int32_t *pslot = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  int32_t *row_of = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  orc_gate_batch(cfg, in, idx, gate, load, psum, NULL);
  const int64_t C = orc_capacity(T, k, n, cfg->capacity_factor);
  orc_dispatch(T, k, n, C, idx, counts, offsets, ptok, pslot, row_of, NULL);
  for (size_t p = 0; p < S; ++p) imp[idx[p]] += gate[p];

  /* the two levels' loads and the group sizes (as the forward sums them) */
  double *cp = (double *)malloc(sizeof(double) * (size_t)mx);
  double *sp = (double *)malloc(sizeof(double) * (size_t)mx);
  double *cs = (double *)malloc(sizeof(double) * (size_t)mx);
  double *ss = (double *)malloc(sizeof(double) * (size_t)mx);
  double *P = (double *)malloc(sizeof(double) * (size_t)mx);
  float *Hp = (float *)malloc(sizeof(float) * (size_t)mx);
  float *Hs = (float *)malloc(sizeof(float) * (size_t)mx);
  int *op = (int *)malloc(sizeof(int) * (size_t)mx);
  int *os = (int *)malloc(sizeof(int) * (size_t)mx);
  double *g1 = (double *)malloc(sizeof(double) * (size_t)(k1 + 1));
  double *g2 = (double *)malloc(sizeof(double) * (size_t)(k2 + 1));
  double *load_p = (double *)calloc((size_t)a, sizeof(double));
  double *load_s = (double *)calloc((size_t)a * b, sizeof(double));
  int64_t *cnt = (int64_t *)calloc((size_t)a, sizeof(int64_t));
  for (int t = 0; t < T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    orc_gate_row(d, a, k1, 0, noise, cfg->seed, (uint32_t)t, 0u, xt, in->Wg, in->bg, in->Wn, cp, sp,
                 Hp, op, g1, NULL, NULL);
    orc_load_row(a, k1, noise, cp, sp, Hp, P);
    for (int i = 0; i < a; ++i) load_p[i] += P[i];
    for (int ps = 0; ps < k1; ++ps) {
      const int gi = op[ps];
      cnt[gi]++;
      orc_gate_row(d, b, k2, 0, noise, cfg->seed, (uint32_t)t, (uint32_t)(1 + gi), xt,
                   in->Wg2 + (size_t)gi * d * b, in->bg2 ? in->bg2 + (size_t)gi * b : NULL,
                   in->Wn2 ? in->Wn2 + (size_t)gi * d * b : NULL, cs, ss, Hs, os, g2, NULL, NULL);
      orc_load_row(b, k2, noise, cs, ss, Hs, P);
      for (int j = 0; j < b; ++j) load_s[(size_t)gi * b + j] += P[j];
    }
  }

  double *lam_imp = (double *)malloc(sizeof(double) * (size_t)n);
  double *lam_load = (double *)malloc(sizeof(double) * (size_t)n);
  orc_cv2_grad(imp, n, lam_imp);
  orc_cv2_grad(load, n, lam_load);
  for (int i = 0; i < n; ++i) {
    lam_imp[i] *= cfg->w_importance;
    lam_load[i] *= cfg->w_load;
  }
  const int load_term = noise && cfg->w_load != 0.0;
  double *lam_p = (double *)calloc((size_t)a, sizeof(double));
  double *lam_s = (double *)calloc((size_t)a * b, sizeof(double));
  for (int i = 0; i < a; ++i) {
    if (cnt[i] == 0) continue;
    for (int j = 0; j < b; ++j) {
      lam_p[i] += lam_load[(size_t)i * b + j] * load_s[(size_t)i * b + j] / (double)cnt[i];
      lam_s[(size_t)i * b + j] = lam_load[(size_t)i * b + j] * load_p[i] / (double)cnt[i];
    }
  }

#define ZERO(ptr, cnt_) do { if (ptr) memset((ptr), 0, sizeof(double) * (size_t)(cnt_)); } while (0)
  ZERO(g->dx, (size_t)T * d);
  ZERO(g->dWg, (size_t)d * a); ZERO(g->dbg, a); ZERO(g->dWn, (size_t)d * a);
  ZERO(g->dWg2, (size_t)a * d * b); ZERO(g->dbg2, (size_t)a * b); ZERO(g->dWn2, (size_t)a * d * b);
  ZERO(g->dW1, (size_t)n * f * d); ZERO(g->db1, (size_t)n * f);
  ZERO(g->dW2, (size_t)n * d * f); ZERO(g->db2, (size_t)n * d);
  ZERO(g->dgate, S);
#undef ZERO
  double *dW1 = g->dW1 ? g->dW1 : (double *)calloc((size_t)n * f * d, sizeof(double));
  double *dW2 = g->dW2 ? g->dW2 : (double *)calloc((size_t)n * d * f, sizeof(double));
  double *dx = g->dx;

  /* ---- combine and experts, as in the flat layer */
  double *dgate = (double *)calloc(S ? S : 1, sizeof(double));
  for (int t = 0; t < T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    const float *dyt = dy + (size_t)t * d;
    double *dxt = dx + (size_t)t * d;
    int kept = 0;
    for (int j = 0; j < k; ++j) {
      size_t pj = (size_t)t * k + j;
      if (row_of[pj] < 0) continue;
      kept++;
      int e = idx[pj];
      dgate[pj] = expert_row_bwd(
          d, f, bf16, xt, (const char *)in->W1 + (size_t)e * f * d * esz,
          in->b1 ? in->b1 + (size_t)e * f : NULL, (const char *)in->W2 + (size_t)e * d * f * esz,
          in->b2 ? in->b2 + (size_t)e * d : NULL, gate[pj], dyt, dW1 + (size_t)e * f * d,
          g->db1 ? g->db1 + (size_t)e * f : NULL, dW2 + (size_t)e * d * f,
          g->db2 ? g->db2 + (size_t)e * d : NULL, dxt);
    }
    if (kept == 0 && cfg->passthrough)
      for (int q = 0; q < d; ++q) dxt[q] += (double)dyt[q];
  }
  if (g->dgate) memcpy(g->dgate, dgate, sizeof(double) * S);

  /* ---- the two gate levels */
  double *dG1 = (double *)malloc(sizeof(double) * (size_t)k1);
  double *dG2 = (double *)malloc(sizeof(double) * (size_t)k2);
  double *dc = (double *)malloc(sizeof(double) * (size_t)mx);
  double *dz = (double *)malloc(sizeof(double) * (size_t)mx);
  double *dH = (double *)malloc(sizeof(double) * (size_t)mx);
  int *rank = (int *)malloc(sizeof(int) * (size_t)mx);
  for (int t = 0; t < T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    double *dxt = dx + (size_t)t * d;
    orc_gate_row(d, a, k1, 0, noise, cfg->seed, (uint32_t)t, 0u, xt, in->Wg, in->bg, in->Wn, cp, sp,
                 Hp, op, g1, NULL, NULL);
    for (int ps = 0; ps < k1; ++ps) dG1[ps] = 0.0;
    for (int ps = 0; ps < k1; ++ps) {
      const int gi = op[ps];
      const float *Wg2 = in->Wg2 + (size_t)gi * d * b;
      const float *Wn2 = in->Wn2 ? in->Wn2 + (size_t)gi * d * b : NULL;
      orc_gate_row(d, b, k2, 0, noise, cfg->seed, (uint32_t)t, (uint32_t)(1 + gi), xt, Wg2,
                   in->bg2 ? in->bg2 + (size_t)gi * b : NULL, Wn2, cs, ss, Hs, os, g2, NULL, NULL);
      /* slot gate G_p G_s: dL/dG_s = dL/dslot G_p, dL/dG_p = sum_ss dL/dslot G_s */
      for (int s2 = 0; s2 < k2; ++s2) {
        const size_t slot = (size_t)t * k + (size_t)ps * k2 + s2;
        const double dslot = dgate[slot] + lam_imp[(size_t)gi * b + os[s2]];
        dG1[ps] += dslot * g2[s2];
        dG2[s2] = dslot * g1[ps];
      }
      level_bwd(b, k2, noise, cfg->seed, (uint32_t)t, (uint32_t)(1 + gi), xt, d, Wn2, cs, ss, Hs, os,
                g2, dG2, load_term ? lam_s + (size_t)gi * b : NULL, dc, dz, dH, rank);
      level_proj_bwd(d, b, noise, xt, Wg2, Wn2, dc, dz, g->dWg2 ? g->dWg2 + (size_t)gi * d * b : NULL,
                     g->dbg2 ? g->dbg2 + (size_t)gi * b : NULL,
                     g->dWn2 ? g->dWn2 + (size_t)gi * d * b : NULL, dxt);
    }
    level_bwd(a, k1, noise, cfg->seed, (uint32_t)t, 0u, xt, d, in->Wn, cp, sp, Hp, op, g1, dG1,
              load_term ? lam_p : NULL, dc, dz, dH, rank);
    /* router z-loss and entropy of the primary gate's clean logits, as flat */
    if (T > 0 && (cfg->w_z != 0.0 || cfg->w_entropy != 0.0)) {
      double m = cp[0];
      for (int i = 1; i < a; ++i) if (cp[i] > m) m = cp[i];
      double Ssum = 0.0;
      for (int i = 0; i < a; ++i) Ssum += exp(cp[i] - m);
      const double logS = log(Ssum);
      double ent = 0.0;
      for (int i = 0; i < a; ++i) {
        const double lp = cp[i] - m - logS;
        ent -= exp(lp) * lp;
      }
      for (int i = 0; i < a; ++i) {
        const double lp = cp[i] - m - logS;
        dc[i] += (cfg->w_z * 2.0 * cp[i] + cfg->w_entropy * exp(lp) * (lp + ent)) / (double)T;
      }
    }
    level_proj_bwd(d, a, noise, xt, in->Wg, in->Wn, dc, dz, g->dWg, g->dbg, g->dWn, dxt);
  }

  if (!g->dW1) free(dW1);
  if (!g->dW2) free(dW2);
  free(dG1); free(dG2); free(dc); free(dz); free(dH); free(rank);
  free(cp); free(sp); free(cs); free(ss); free(P); free(Hp); free(Hs); free(op); free(os);
  free(g1); free(g2); free(load_p); free(load_s); free(cnt); free(lam_p); free(lam_s);
  free(lam_imp); free(lam_load); free(dgate);
  free(idx); free(gate); free(load); free(psum); free(imp); free(counts); free(offsets);
  free(ptok); free(pslot); free(row_of);
  return 0;
}

int orc_backward(const orc_cfg *cfg, const orc_inputs *in, const float *dy, orc_grads *g)
{
  if (!valid_cfg(cfg)) return -1;
  if (cfg->hier_a) return cfg->shared_expert ? -1 : orc_backward_hier(cfg, in, dy, g);
  if (cfg->shared_expert && (!in->W1s || !in->W2s)) return -1;
  const int T = cfg->T, d = cfg->d, n = cfg->n, k = cfg->k, f = cfg->f, bf16 = cfg->expert_bf16;
  const int noise = cfg->noise;
  const size_t esz = bf16 ? 2 : 4;
  const size_t S = (size_t)T * k;

  /* ---- forward state: routing, dispatch, importance, load */
  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  double *gate = (double *)malloc(sizeof(double) * (S ? S : 1));
  double *load = (double *)malloc(sizeof(double) * (size_t)n);
  double *psum = (double *)malloc(sizeof(double) * (size_t)n);
  double *imp = (double *)calloc((size_t)n, sizeof(double));
  int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
  int32_t *ptok = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  int32_t *pslot = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  int32_t *row_of = (int32_t *)malloc(sizeof(int32_t) * (S ? S : 1));
  orc_gate_batch(cfg, in, idx, gate, load, psum, NULL);
  const int64_t C = orc_capacity(T, k, n, cfg->capacity_factor);
  orc_dispatch(T, k, n, C, idx, counts, offsets, ptok, pslot, row_of, NULL);
  for (size_t p = 0; p < S; ++p) imp[idx[p]] += gate[p];

  /* ---- the losses' gradients with respect to Importance and Load */
  double *lam_imp = (double *)malloc(sizeof(double) * (size_t)n);
  double *lam_load = (double *)malloc(sizeof(double) * (size_t)n);
  orc_cv2_grad(imp, n, lam_imp);
  orc_cv2_grad(load, n, lam_load);
  for (int i = 0; i < n; ++i) {
    lam_imp[i] *= cfg->w_importance;
    lam_load[i] *= cfg->w_load;
  }

  /* ---- zero the outputs */
#define ZERO(ptr, cnt) do { if (ptr) memset((ptr), 0, sizeof(double) * (size_t)(cnt)); } while (0)
  ZERO(g->dx, (size_t)T * d);
  ZERO(g->dWg, (size_t)d * n); ZERO(g->dbg, n); ZERO(g->dWn, (size_t)d * n);
  ZERO(g->dW1, (size_t)n * f * d); ZERO(g->db1, (size_t)n * f);
  ZERO(g->dW2, (size_t)n * d * f); ZERO(g->db2, (size_t)n * d);
  ZERO(g->dW1s, (size_t)f * d); ZERO(g->db1s, f); ZERO(g->dW2s, (size_t)d * f); ZERO(g->db2s, d);
  ZERO(g->dgate, S); ZERO(g->dlogits, (size_t)T * n); ZERO(g->dnoise, (size_t)T * n);
#undef ZERO
  double *dW1 = g->dW1 ? g->dW1 : (double *)calloc((size_t)n * f * d, sizeof(double));
  double *dW2 = g->dW2 ? g->dW2 : (double *)calloc((size_t)n * d * f, sizeof(double));
  double *dW1s = NULL, *dW2s = NULL;
  if (cfg->shared_expert) {
    dW1s = g->dW1s ? g->dW1s : (double *)calloc((size_t)f * d, sizeof(double));
    dW2s = g->dW2s ? g->dW2s : (double *)calloc((size_t)d * f, sizeof(double));
  }
  double *dx = g->dx;

  /* ---- combine and experts: y_t = sum_j g_tj E_{e_tj}(x_t) (+ E_shared(x_t)) */
  double *dgate = (double *)calloc(S ? S : 1, sizeof(double));
  for (int t = 0; t < T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    const float *dyt = dy + (size_t)t * d;
    double *dxt = dx + (size_t)t * d;
    int kept = 0;
    for (int j = 0; j < k; ++j) {
      size_t pj = (size_t)t * k + j;
      if (row_of[pj] < 0) continue; /* dropped: contributes nothing */
      kept++;
      int e = idx[pj];
      dgate[pj] = expert_row_bwd(
          d, f, bf16, xt, (const char *)in->W1 + (size_t)e * f * d * esz,
          in->b1 ? in->b1 + (size_t)e * f : NULL, (const char *)in->W2 + (size_t)e * d * f * esz,
          in->b2 ? in->b2 + (size_t)e * d : NULL, gate[pj], dyt, dW1 + (size_t)e * f * d,
          g->db1 ? g->db1 + (size_t)e * f : NULL, dW2 + (size_t)e * d * f,
          g->db2 ? g->db2 + (size_t)e * d : NULL, dxt);
    }
    if (kept == 0 && cfg->passthrough)
      for (int q = 0; q < d; ++q) dxt[q] += (double)dyt[q]; /* y = x */
    if (cfg->shared_expert)
      expert_row_bwd(d, f, bf16, xt, in->W1s, in->b1s, in->W2s, in->b2s, 1.0, dyt, dW1s, g->db1s,
                     dW2s, g->db2s, dxt);
  }
  if (g->dgate) memcpy(g->dgate, dgate, sizeof(double) * S);

  /* ---- gate */
  double *c = (double *)malloc(sizeof(double) * (size_t)n);
  double *s = (double *)malloc(sizeof(double) * (size_t)n);
  double *pr = (double *)malloc(sizeof(double) * (size_t)n);
  double *gk = (double *)malloc(sizeof(double) * (size_t)k);
  double *dG = (double *)malloc(sizeof(double) * (size_t)k);
  double *dc = (double *)malloc(sizeof(double) * (size_t)n);
  double *ds = (double *)malloc(sizeof(double) * (size_t)n);
  double *dH = (double *)malloc(sizeof(double) * (size_t)n);
  double *zp = (double *)malloc(sizeof(double) * (size_t)n);
  float *H = (float *)malloc(sizeof(float) * (size_t)n);
  int *order = (int *)malloc(sizeof(int) * (size_t)n);
  int *rank = (int *)malloc(sizeof(int) * (size_t)n);
  for (int t = 0; t < T; ++t) {
    const float *xt = in->x + (size_t)t * d;
    orc_gate_row(d, n, k, cfg->router, noise, cfg->seed, (uint32_t)t, 0u, xt, in->Wg, in->bg,
                 in->Wn, c, s, H, order, gk, pr, in->sel_bias);
    for (int r = 0; r < n; ++r) rank[order[r]] = r;
    for (int i = 0; i < n; ++i) dc[i] = ds[i] = dH[i] = 0.0;
    /* dL/dG of each kept gate: from the combine, and from Importance (the sum
     * of the gates, dropped slots included) */
    for (int j = 0; j < k; ++j) dG[j] = dgate[(size_t)t * k + j] + lam_imp[order[j]];

    if (cfg->router == 0) {
      /* G = Softmax over the kept k of H: dH_i = G_i (dG_i - sum_l G_l dG_l) */
      double sum = 0.0;
      for (int j = 0; j < k; ++j) sum += gk[j] * dG[j];
      for (int j = 0; j < k; ++j) dH[order[j]] = gk[j] * (dG[j] - sum);
    } else if (cfg->router == 1) {
      /* gate = p_argmax of p = softmax(c); the auxiliary loss
       * alpha N sum_i f_i P_i has dP_i/dp_ti = 1/T with f_i fixed */
      double *dp = dH; /* reuse: router 1 has no H gradient of its own */
      for (int i = 0; i < n; ++i)
        dp[i] = T > 0 ? cfg->alpha * (double)n * ((double)counts[i] / (double)T) / (double)T : 0.0;
      dp[order[0]] += dG[0];
      double sum = 0.0;
      for (int i = 0; i < n; ++i) sum += pr[i] * dp[i];
      for (int i = 0; i < n; ++i) dc[i] += pr[i] * (dp[i] - sum);
      for (int i = 0; i < n; ++i) dH[i] = 0.0;
    } else {
      /* router 2: g_j = sigma(c_j) / S, S = sum over the kept of sigma:
       * d sigma_m = (dG_m - sum_j g_j dG_j) / S, d c = d sigma * sigma (1 - sigma) */
      double Ssum = 0.0, sum = 0.0;
      for (int j = 0; j < k; ++j) Ssum += 1.0 / (1.0 + exp(-c[order[j]]));
      for (int j = 0; j < k; ++j) sum += gk[j] * dG[j];
      for (int j = 0; j < k; ++j) {
        double sg = 1.0 / (1.0 + exp(-c[order[j]]));
        dc[order[j]] += (dG[j] - sum) / Ssum * sg * (1.0 - sg);
      }
    }

    if (noise && cfg->w_load != 0.0) {
      /* P(x,i) = Phi((c_i - thr_i) / s_i), thr_i = H of the (k+1)-th ranked
       * expert when i is kept, else of the k-th; Load_i = sum_t P(x_t,i) */
      const int jk = order[k - 1], jk1 = k < n ? order[k] : -1;
      for (int i = 0; i < n; ++i) {
        const int jt = rank[i] < k ? jk1 : jk;
        if (jt < 0 || s[i] == 0.0) continue; /* P is constant there */
        const double u = (c[i] - (double)H[jt]) / s[i];
        const double dens = exp(-0.5 * u * u) / sqrt(2.0 * acos(-1.0));
        const double a = lam_load[i] * dens / s[i];
        dc[i] += a;
        ds[i] -= a * u;
        dH[jt] -= a;
      }
    }
    /* router z-loss w_z mean_t |c_t|^2 and gate entropy -w_entropy mean_t
     * H(softmax(c_t)) ([MoE-intro] 第三部分): d|c|^2/dc_i = 2 c_i;
     * dH/dc_i = -p_i (log p_i + H) for p = softmax(c) */
    if (T > 0 && (cfg->w_z != 0.0 || cfg->w_entropy != 0.0)) {
      double m = c[0];
      for (int i = 1; i < n; ++i) if (c[i] > m) m = c[i];
      double Ssum = 0.0;
      for (int i = 0; i < n; ++i) Ssum += exp(c[i] - m);
      const double logS = log(Ssum);
      double ent = 0.0;
      for (int i = 0; i < n; ++i) {
        const double lp = c[i] - m - logS;
        ent -= exp(lp) * lp;
      }
      for (int i = 0; i < n; ++i) {
        const double lp = c[i] - m - logS;
        dc[i] += (cfg->w_z * 2.0 * c[i] + cfg->w_entropy * exp(lp) * (lp + ent)) / (double)T;
      }
    }
    /* H = c + eps * s (noise), H = c otherwise (router 2's bias has no gradient) */
    for (int i = 0; i < n; ++i) {
      dc[i] += dH[i];
      if (noise) ds[i] += dH[i] * orc_noise(cfg->seed, (uint32_t)t, (uint32_t)i, 0u);
    }
    /* s = Softplus(z), z = x W_noise: dz = ds * Sigmoid(z) */
    if (noise) {
      for (int i = 0; i < n; ++i) zp[i] = 0.0;
      for (int q = 0; q < d; ++q)
        for (int i = 0; i < n; ++i) zp[i] += (double)xt[q] * (double)in->Wn[(size_t)q * n + i];
      for (int i = 0; i < n; ++i) ds[i] *= 1.0 / (1.0 + exp(-zp[i]));
    }
    if (g->dlogits) memcpy(g->dlogits + (size_t)t * n, dc, sizeof(double) * (size_t)n);
    if (g->dnoise && noise) memcpy(g->dnoise + (size_t)t * n, ds, sizeof(double) * (size_t)n);
    /* c = x W_g + b_g, z = x W_noise */
    double *dxt = dx + (size_t)t * d;
    for (int q = 0; q < d; ++q) {
      double acc = 0.0;
      for (int i = 0; i < n; ++i) {
        acc += in->Wg[(size_t)q * n + i] * dc[i];
        if (g->dWg) g->dWg[(size_t)q * n + i] += (double)xt[q] * dc[i];
        if (noise) {
          acc += in->Wn[(size_t)q * n + i] * ds[i];
          if (g->dWn) g->dWn[(size_t)q * n + i] += (double)xt[q] * ds[i];
        }
      }
      dxt[q] += acc;
    }
    if (g->dbg)
      for (int i = 0; i < n; ++i) g->dbg[i] += dc[i];
  }

  if (!g->dW1) free(dW1);
  if (!g->dW2) free(dW2);
  if (cfg->shared_expert && !g->dW1s) free(dW1s);
  if (cfg->shared_expert && !g->dW2s) free(dW2s);
  free(c); free(s); free(pr); free(gk); free(dG); free(dc); free(ds); free(dH); free(zp);
  free(H); free(order); free(rank); free(dgate);
  free(idx); free(gate); free(load); free(psum); free(imp); free(counts); free(offsets);
  free(ptok); free(pslot); free(row_of); free(lam_imp); free(lam_load);
  return 0;
}
