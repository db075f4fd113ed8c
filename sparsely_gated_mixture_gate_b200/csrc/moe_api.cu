// moe_api.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace layout, the launch sequence of every entry point, and tracing.
// Host code only; the arithmetic is in the kernels of the other files.
#include <limits.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace moe {

// ---------------------------------------------------------------- side stream
namespace {
// moe_forward runs the balance statistics (the reduction of the smoothed Load,
// Importance and the losses) on a second stream beside the dispatch -> experts
// -> combine chain: they feed only the loss outputs.  Fork and join are
// events, so the whole call stays ordered on the caller's stream.  One stream
// and its events per device and host thread, so concurrent callers on other
// threads never wait on one another's events.
struct Side {
  cudaStream_t s = nullptr;
  cudaEvent_t fork_gate = nullptr, fork_dispatch = nullptr, join = nullptr;
};
thread_local std::vector<Side> t_side;  // by device

bool is_side_stream(cudaStream_t st) {
  for (const auto &sd : t_side)
    if (sd.s && sd.s == st) return true;
  return false;
}
}  // namespace

// ---------------------------------------------------------------- tracing
namespace {
struct TraceRec {
  const char *name;
  cudaEvent_t a, b;
  bool side;  // launched on the side stream: its time overlaps the main chain
};
struct TraceAgg {
  std::string name;
  int launches;
  double ms;
};
bool g_trace = false;
std::vector<TraceRec> g_pending;
std::vector<cudaEvent_t> g_pool;
std::vector<TraceAgg> g_agg;
long long g_launches = 0;

cudaEvent_t pooled_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void trace_collect() {
  for (auto &r : g_pending) {
    float ms = 0.f;
    cudaEventSynchronize(r.b);
    cudaEventElapsedTime(&ms, r.a, r.b);
    bool found = false;
    const std::string name = r.side ? std::string(r.name) + " [side stream]" : std::string(r.name);
    for (auto &g : g_agg)
      if (g.name == name) {
        g.launches += 1;
        g.ms += ms;
        found = true;
        break;
      }
    if (!found) g_agg.push_back({name, 1, (double)ms});
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_pending.clear();
}
}  // namespace

void trace_begin(const char *name, cudaStream_t st, int *slot) {
  if (!g_trace) return;
  TraceRec r{name, pooled_event(), pooled_event(), is_side_stream(st)};
  cudaEventRecord(r.a, st);
  g_pending.push_back(r);
  *slot = (int)g_pending.size() - 1;
}
void trace_end(int slot, cudaStream_t st) {
  if (slot >= 0) cudaEventRecord(g_pending[slot].b, st);
}
void count_launch() { ++g_launches; }

int num_sms() {
  static PerDevice sms;
  int v = 148;
  sms.get([](int dev, int *out) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c < 1)
      return MOE_EDEVICE;
    *out = c;
    return MOE_OK;
  }, &v);
  return v;
}

int check_device() {
  static PerDevice checked;
  return checked.get([](int dev, int *) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_EDEVICE;
    return (major == 10 && minor == 0) ? MOE_OK : MOE_EDEVICE;  // built for sm_100a only
  });
}

int route_rows_per_tile(int R) {
  // about eight routing tiles per SM of a 148-SM part, 4..256 rows each
  int64_t rt = ceil_div(R, 1184);
  rt = ceil_div(rt, 4) * 4;
  if (rt < 4) rt = 4;
  if (rt > 256) rt = 256;
  return (int)rt;
}

// ---------------------------------------------------------------- workspace layout
namespace {

struct Layout {
  size_t c, s, c2, s2, load_part, psum_part, prob_sum;
  size_t stats_part, rstats;  // router statistics: per-tile sums, their totals
  size_t pidx, pgate, load_p, g_hist, g_base, g_counts, g_offsets, g_ucoff, g_perm_token,
      g_perm_slot, g_row_of, g_mblk, g_tiles, load2_part, load2;
  size_t hist, base, ucoff, offsets, perm_token, row_of, gate_sorted, counts_scratch, ticket;
  size_t mprefix, tab1, tab2, mdone, x_perm, hid, y_perm;
  size_t x_shared, y_shared, shared_off;  // shared expert: input and output rows, {0, T}
  size_t shared_mprefix, shared_tab1, shared_tab2, shared_mdone;  // and its GEMM plan
  size_t xhi, xlo, whi, wlo;  // three-pass TF32 gate operands
  // backward pass (cfg.backward): the forward's extra state, then scratch
  size_t kth, hid_shared;
  size_t dy_perm, dhid, dx_perm, dy_shared, dhid_shared, dx_shared, dgate, lam_imp, lam_load,
      sw_coef, dc, dz, colsum_part, sgemm_part;
  // hierarchical backward: the secondary rows' thresholds, own gates and ids,
  // the two levels' gate gradients and load coefficients, the secondary
  // logits' gradients, and each secondary row's part of dx
  size_t kth2, gate2, idx2, dgp, dgs, lam_p, lam_s, dc2, dz2, dxs;
  size_t total;
  int RT1, tiles1, RT2, tiles2_upper, B;
};

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t at = off;
    off += (bytes + 255) & ~(size_t)255;
    return at;
  }
};

Layout make_layout(const moe_config &c) {
  Layout L;
  Bump bp;
  const size_t T = (size_t)c.T, n = (size_t)c.n, k = (size_t)c.k;
  const bool hier = c.hier_a > 0;
  const size_t ng = hier ? (size_t)c.hier_a : n;
  const size_t S = T * k;
  const size_t esz = c.expert_dtype == MOE_BF16 ? 2 : 4;
  L.RT1 = route_rows_per_tile(c.T);
  L.tiles1 = (int)ceil_div(c.T, L.RT1);
  size_t R2 = 0;
  if (hier) {
    R2 = T * (size_t)c.hier_k1;
    L.RT2 = route_rows_per_tile((int)R2);
    L.tiles2_upper = (int)ceil_div((int64_t)R2, L.RT2) + c.hier_a;
  } else {
    L.RT2 = 0;
    L.tiles2_upper = 0;
  }
  // the flat / primary gate's logits; a hierarchical layer's secondary gates
  // have their own (the backward reads both levels)
  L.c = bp.take(4 * T * ng);
  L.s = bp.take(4 * T * ng);
  L.c2 = hier ? bp.take(4 * R2 * (size_t)c.hier_b) : 0;
  L.s2 = hier ? bp.take(4 * R2 * (size_t)c.hier_b) : 0;
  const size_t lp1 = (size_t)L.tiles1 * ng, lp2 = (size_t)L.tiles2_upper * (size_t)c.hier_b;
  L.load_part = bp.take(4 * lp1);
  L.psum_part = bp.take(c.router == MOE_ROUTER_SWITCH ? 4 * (size_t)L.tiles1 * n : 0);
  L.prob_sum = bp.take(4 * n);
  L.stats_part = bp.take(c.router_stats ? 8 * (size_t)L.tiles1 : 0);
  L.rstats = bp.take(c.router_stats ? 8 : 0);
  L.B = (int)ceil_div(c.T, dispatch_tokens_per_block(c.T));
  if (hier) {
    const size_t a = (size_t)c.hier_a, k1 = (size_t)c.hier_k1;
    L.pidx = bp.take(4 * T * k1);
    L.pgate = bp.take(4 * T * k1);
    L.load_p = bp.take(4 * a);
    L.g_hist = bp.take(4 * (size_t)L.B * a);
    L.g_base = bp.take(4 * (size_t)L.B * a);
    L.g_counts = bp.take(4 * a);
    L.g_offsets = bp.take(4 * (a + 1));
    L.g_ucoff = bp.take(4 * (a + 1));
    L.g_perm_token = bp.take(4 * T * k1);
    L.g_perm_slot = bp.take(4 * T * k1);
    L.g_row_of = bp.take(4 * T * k1);
    L.g_mblk = bp.take(4 * (a + 1));
    L.g_tiles = bp.take(4 * (a + 1));
    // its own buffer: both levels' partial sums are reduced after the secondary routing
    L.load2_part = bp.take(4 * lp2);
    L.load2 = bp.take(4 * n);
  } else {
    L.pidx = L.pgate = L.load_p = L.g_hist = L.g_base = L.g_counts = L.g_offsets = L.g_ucoff =
        L.g_perm_token = L.g_perm_slot = L.g_row_of = L.g_mblk = L.g_tiles = L.load2_part =
            L.load2 = 0;
  }
  L.hist = bp.take(4 * (size_t)L.B * n);
  L.base = bp.take(4 * (size_t)L.B * n);
  L.ucoff = bp.take(4 * (n + 1));
  L.offsets = bp.take(4 * (n + 1));
  L.perm_token = bp.take(4 * S);
  L.row_of = bp.take(4 * S);
  L.gate_sorted = bp.take(4 * S);
  L.counts_scratch = bp.take(4 * n);
  L.ticket = bp.take(4);
  L.mprefix = bp.take(4 * (n + 1));
  {
    const size_t mb_upper = (size_t)ceil_div((int64_t)S, kExpertBM) + n;
    L.tab1 = bp.take(16 * mb_upper * (size_t)ceil_div(c.f, kExpertBN));
    L.tab2 = bp.take(16 * mb_upper * (size_t)ceil_div(c.d, kExpertBN));
    L.mdone = bp.take(4 * (mb_upper + 1));
  }
  L.x_perm = bp.take(esz * S * (size_t)c.d);
  L.hid = bp.take(esz * S * (size_t)c.f);
  L.y_perm = bp.take(esz * S * (size_t)c.d);
  if (c.shared_expert) {
    L.x_shared = bp.take(esz * (size_t)T * c.d);
    L.y_shared = bp.take(esz * (size_t)T * c.d);
    L.shared_off = bp.take(8);
    const size_t mbe = (size_t)ceil_div((int64_t)T, kExpertBM);
    L.shared_mprefix = bp.take(8);
    L.shared_tab1 = bp.take(16 * mbe * (size_t)ceil_div(c.f, kExpertBN));
    L.shared_tab2 = bp.take(16 * mbe * (size_t)ceil_div(c.d, kExpertBN));
    L.shared_mdone = bp.take(4 * (mbe + 1));
  } else {
    L.x_shared = L.y_shared = L.shared_off = 0;
    L.shared_mprefix = L.shared_tab1 = L.shared_tab2 = L.shared_mdone = 0;
  }
  if (c.gate_precision == MOE_GATE_TF32X3) {
    const size_t rows = hier ? (T > R2 ? T : R2) : T;
    const size_t nw = (size_t)(c.noise ? 2 : 1);
    const size_t wr1 = nw * ng, wr2 = hier ? nw * (size_t)c.hier_a * c.hier_b : 0;
    const size_t wrows = wr1 > wr2 ? wr1 : wr2;
    L.xhi = bp.take(4 * rows * (size_t)c.d);
    L.xlo = bp.take(4 * rows * (size_t)c.d);
    L.whi = bp.take(4 * wrows * (size_t)c.d);
    L.wlo = bp.take(4 * wrows * (size_t)c.d);
  } else {
    L.xhi = L.xlo = L.whi = L.wlo = 0;
  }
  L.kth = L.hid_shared = L.dy_perm = L.dhid = L.dx_perm = L.dy_shared = L.dhid_shared =
      L.dx_shared = L.dgate = L.lam_imp = L.lam_load = L.sw_coef = L.dc = L.dz = L.colsum_part =
          L.sgemm_part = 0;
  L.kth2 = L.gate2 = L.idx2 = L.dgp = L.dgs = L.lam_p = L.lam_s = L.dc2 = L.dz2 = L.dxs = 0;
  if (c.backward) {
    L.kth = bp.take(16 * T);
    L.hid_shared = bp.take(c.shared_expert ? esz * T * (size_t)c.f : 0);
    L.dy_perm = bp.take(esz * S * (size_t)c.d);
    L.dhid = bp.take(esz * S * (size_t)c.f);
    L.dx_perm = bp.take(esz * S * (size_t)c.d);
    if (c.shared_expert) {
      L.dy_shared = bp.take(esz * T * (size_t)c.d);
      L.dhid_shared = bp.take(esz * T * (size_t)c.f);
      L.dx_shared = bp.take(esz * T * (size_t)c.d);
    }
    L.dgate = bp.take(4 * S);
    L.lam_imp = bp.take(4 * n);
    L.lam_load = bp.take(4 * n);
    L.sw_coef = bp.take(4 * n);
    L.dc = bp.take(4 * T * ng);
    L.dz = bp.take(c.noise ? 4 * T * ng : 0);
    L.colsum_part = bp.take(4 * (size_t)colsum_parts(c.T, (int)ng) * ng);
    const size_t np = c.noise ? 2 : 1;  // dW_g, and dW_noise beside it
    const size_t sp = (size_t)sgemm_splits(c.d, (int)ng, c.T, (int)np);
    L.sgemm_part = bp.take(sp > 1 ? 4 * np * sp * (size_t)c.d * ng : 0);
    if (hier) {
      const size_t a = (size_t)c.hier_a, b = (size_t)c.hier_b;
      const size_t k1 = (size_t)c.hier_k1, k2 = (size_t)c.hier_k2;
      L.kth2 = bp.take(16 * R2);
      L.gate2 = bp.take(4 * R2 * k2);
      L.idx2 = bp.take(4 * R2 * k2);
      L.dgp = bp.take(4 * T * k1);
      L.dgs = bp.take(4 * R2 * k2);
      L.lam_p = bp.take(4 * a);
      L.lam_s = bp.take(4 * a * b);
      L.dc2 = bp.take(4 * R2 * b);
      L.dz2 = bp.take(c.noise ? 4 * R2 * b : 0);
      L.dxs = bp.take(4 * R2 * (size_t)c.d);
    }
  }
  L.total = bp.off;
  return L;
}

template <class P>
P *at(void *ws, size_t off) {
  return reinterpret_cast<P *>(static_cast<char *>(ws) + off);
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int64_t capacity_of(const moe_config &c) {
  if (!(c.capacity_factor > 0.0)) return INT64_MAX;
  return (int64_t)ceil((double)c.T * (double)c.k * c.capacity_factor / (double)c.n);
}


int common_checks(const moe_config *cfg, void *ws, size_t ws_bytes, int32_t *status,
                  Layout *L) {
  const int v = moe_validate(cfg);
  if (v != MOE_OK) return v;
  if (!status) return MOE_EINVAL;
  *L = make_layout(*cfg);
  if (ws_bytes < L->total) return MOE_EWORKSPACE;
  if (L->total > 0 && (!ws || !aligned(ws, 256))) return MOE_EWORKSPACE;
  return check_device();
}

// ---------------------------------------------------------------- side stream
int side_stream(Side **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ECUDA;
  if ((int)t_side.size() <= dev) t_side.resize(dev + 1);
  Side &sd = t_side[dev];
  if (!sd.s) {
    cudaStream_t s = nullptr;
    cudaEvent_t e[3] = {nullptr, nullptr, nullptr};
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return MOE_ECUDA;
    for (auto &ev : e)
      if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return MOE_ECUDA;
    sd.fork_gate = e[0];
    sd.fork_dispatch = e[1];
    sd.join = e[2];
    sd.s = s;
  }
  *out = &sd;
  return MOE_OK;
}

// work queued on `to` after this waits for everything queued on `from` so far
int stream_after(cudaStream_t to, cudaStream_t from, cudaEvent_t ev) {
  if (cudaEventRecord(ev, from) != cudaSuccess) return MOE_ECUDA;
  if (cudaStreamWaitEvent(to, ev, 0) != cudaSuccess) return MOE_ECUDA;
  return MOE_OK;
}

// ---------------------------------------------------------------- stage drivers
// side: when given, the flat gate's Load (and Switch P) reductions go there
int run_gate(const moe_config &c, const Layout &L, const float *x, const moe_gate_params &gp,
             int *idx, float *gate, float *load, float *prob_sum, void *ws, int *status,
             cudaStream_t st, const Side *side = nullptr) {
  if (c.T == 0) {
    if (cudaMemsetAsync(load, 0, 4 * (size_t)c.n, st) != cudaSuccess) return MOE_ECUDA;
    if (prob_sum && cudaMemsetAsync(prob_sum, 0, 4 * (size_t)c.n, st) != cudaSuccess)
      return MOE_ECUDA;
    return MOE_OK;
  }
  float *cbuf = at<float>(ws, L.c), *sbuf = at<float>(ws, L.s);
  const bool hier = c.hier_a > 0;
  const int ng = hier ? c.hier_a : c.n;

  GateGemmArgs g{};
  g.x = x;
  g.d = c.d;
  g.R = c.T;
  g.G = 1;
  g.Wg = gp.W_g;
  g.Wn = gp.W_noise;
  g.bias = gp.b_g;
  g.nb = ng;
  g.noise = c.noise;
  g.c = cbuf;
  g.s = sbuf;
  g.status = status;
  auto gate_gemm = [&](const GateGemmArgs &ga, int mblk_upper) -> int {
    if (c.gate_precision == MOE_GATE_TF32X3)
      return launch_gate_tf32x3(ga, mblk_upper, at<float>(ws, L.xhi), at<float>(ws, L.xlo),
                                at<float>(ws, L.whi), at<float>(ws, L.wlo), st);
    return launch_gate_gemm(ga, mblk_upper, st);
  };
  MOE_TRY(gate_gemm(g, (int)ceil_div(c.T, kGateBM)));

  RouteArgs r{};
  r.c = cbuf;
  r.s = sbuf;
  r.R = c.T;
  r.nb = ng;
  r.router = c.router;
  r.noise = c.noise;
  r.seed = c.seed;
  r.token_base = (uint32_t)c.token_base;
  r.seed_dev = reinterpret_cast<const unsigned long long *>(gp.seed_dev);
  r.G = 1;
  r.RT = L.RT1;
  r.load_part = at<float>(ws, L.load_part);
  r.sel_bias = (!hier && c.router == MOE_ROUTER_SIGMOID) ? gp.sel_bias : nullptr;
  r.stats_part = c.router_stats ? at<float>(ws, L.stats_part) : nullptr;  // flat / primary rows
  r.kth = c.backward ? at<int4>(ws, L.kth) : nullptr;  // flat / primary rows
  r.status = status;
  if (!hier) {
    r.k = c.k;
    r.out_idx = idx;
    r.out_gate = gate;
    r.K = c.k;
    const bool sw = c.router == MOE_ROUTER_SWITCH;
    r.psum_part = sw ? at<float>(ws, L.psum_part) : nullptr;
    MOE_TRY(launch_route(r, L.tiles1, st));
    cudaStream_t rs = st;
    if (side) {
      MOE_TRY(stream_after(side->s, st, side->fork_gate));
      rs = side->s;
    }
    MOE_TRY(launch_route_reduce(r.load_part, nullptr, 1, L.tiles1, c.n, load, rs));
    if (r.stats_part)
      MOE_TRY(launch_route_reduce(r.stats_part, nullptr, 1, L.tiles1, 2, at<float>(ws, L.rstats), rs));
    if (sw) {
      float *ps = prob_sum ? prob_sum : at<float>(ws, L.prob_sum);
      MOE_TRY(launch_route_reduce(r.psum_part, nullptr, 1, L.tiles1, c.n, ps, rs));
    } else if (prob_sum) {
      if (cudaMemsetAsync(prob_sum, 0, 4 * (size_t)c.n, rs) != cudaSuccess) return MOE_ECUDA;
    }
    return MOE_OK;
  }

  // ---- hierarchical: primary gate over groups
  const int a = c.hier_a, b = c.hier_b, k1 = c.hier_k1, k2 = c.hier_k2;
  int *pidx = at<int>(ws, L.pidx);
  float *pgate = at<float>(ws, L.pgate);
  r.k = k1;
  r.out_idx = pidx;
  r.out_gate = pgate;
  r.K = k1;
  MOE_TRY(launch_route(r, L.tiles1, st));
  // (the primary gate's Load and statistics are reduced below, with the secondary Load)

  // ---- tokens grouped by their kept groups (stable), tile prefixes per group
  DispatchArgs da{};
  da.idx = pidx;
  da.T = c.T;
  da.k = k1;
  da.n = a;
  da.C = INT64_MAX;
  da.hist = at<int>(ws, L.g_hist);
  da.base = at<int>(ws, L.g_base);
  da.ticket = at<int>(ws, L.ticket);
  da.counts = at<int>(ws, L.g_counts);
  da.offsets = at<int>(ws, L.g_offsets);
  da.ucoff = at<int>(ws, L.g_ucoff);
  da.perm_token = at<int>(ws, L.g_perm_token);
  da.perm_slot = at<int>(ws, L.g_perm_slot);
  da.row_of = at<int>(ws, L.g_row_of);
  da.seg_mblk = at<int>(ws, L.g_mblk);
  da.mblk_rows = kGateBM;
  da.seg_tiles = at<int>(ws, L.g_tiles);
  da.tile_rows = L.RT2;
  da.status = status;
  MOE_TRY(launch_dispatch(da, st));

  // ---- secondary gates: grouped fp32 GEMM over each group's tokens
  const int R2 = c.T * k1;
  GateGemmArgs g2 = g;
  g2.c = at<float>(ws, L.c2);
  g2.s = at<float>(ws, L.s2);
  g2.row_token = da.perm_token;
  g2.seg_off = da.offsets;
  g2.seg_mblk = da.seg_mblk;
  g2.R = R2;
  g2.G = a;
  g2.Wg = gp.W_g2;
  g2.Wn = gp.W_noise2;
  g2.bias = gp.b_g2;
  g2.nb = b;
  MOE_TRY(gate_gemm(g2, (int)ceil_div(R2, kGateBM) + a));

  RouteArgs r2 = r;
  r2.stats_part = nullptr;  // the statistics cover the primary gate only
  r2.c = g2.c;
  r2.s = g2.s;
  r2.kth = c.backward ? at<int4>(ws, L.kth2) : nullptr;
  r2.gate_raw = c.backward ? at<float>(ws, L.gate2) : nullptr;
  r2.idx_raw = c.backward ? at<int>(ws, L.idx2) : nullptr;
  r2.R = R2;
  r2.nb = b;
  r2.k = k2;
  r2.router = MOE_ROUTER_NOISY_TOPK;
  r2.row_token = da.perm_token;
  r2.row_slot = da.perm_slot;
  r2.seg_off = da.offsets;
  r2.seg_tiles = da.seg_tiles;
  r2.G = a;
  r2.RT = L.RT2;
  r2.secondary = 1;
  r2.out_idx = idx;
  r2.out_gate = gate;
  r2.K = c.k;
  r2.expert_stride = b;
  r2.gate_mult = pgate;
  r2.k1 = k1;
  r2.load_part = at<float>(ws, L.load2_part);
  r2.psum_part = nullptr;
  MOE_TRY(launch_route(r2, L.tiles2_upper, st));
  // the Load of both levels and the statistics feed only the balancing losses:
  // with a side stream they are reduced there, off the dispatch -> experts chain
  cudaStream_t rs = st;
  if (side) {
    MOE_TRY(stream_after(side->s, st, side->fork_gate));
    rs = side->s;
  }
  MOE_TRY(launch_route_reduce(r.load_part, nullptr, 1, L.tiles1, a, at<float>(ws, L.load_p), rs));
  if (r.stats_part)
    MOE_TRY(launch_route_reduce(r.stats_part, nullptr, 1, L.tiles1, 2, at<float>(ws, L.rstats), rs));
  MOE_TRY(launch_route_reduce(r2.load_part, da.seg_tiles, a, 0, b, at<float>(ws, L.load2), rs));
  MOE_TRY(launch_hier_load(at<float>(ws, L.load_p), at<float>(ws, L.load2), da.counts, a, b, load,
                           rs));
  if (prob_sum && cudaMemsetAsync(prob_sum, 0, 4 * (size_t)c.n, rs) != cudaSuccess)
    return MOE_ECUDA;
  return MOE_OK;
}

// x / x_perm: when x is given its rows are copied into their expert rows
int run_dispatch(const moe_config &c, const Layout &L, const int *idx, const float *gate,
                 int64_t C, int *counts, int *offsets, int *perm_token, int *row_of,
                 const float *x, void *x_perm, void *ws, int *status, cudaStream_t st,
                 bool plan_experts = false, void *x_shared = nullptr, int *shared_off = nullptr) {
  DispatchArgs da{};
  da.x_shared = x_shared;
  da.shared_off = shared_off;
  if (shared_off) {
    da.shared_mprefix = at<int>(ws, L.shared_mprefix);
    da.shared_tab1 = at<int4>(ws, L.shared_tab1);
    da.shared_tab2 = at<int4>(ws, L.shared_tab2);
    da.shared_mdone = at<int>(ws, L.shared_mdone);
    da.nblk1 = (int)ceil_div(c.f, kExpertBN);
    da.nblk2 = (int)ceil_div(c.d, kExpertBN);
  }
  da.ticket = at<int>(ws, L.ticket);
  da.x = x;
  da.x_perm = x_perm;
  da.d = c.d;
  da.x_bf16 = c.expert_dtype == MOE_BF16;
  da.idx = idx;
  da.T = c.T;
  da.k = c.k;
  da.n = c.n;
  da.C = C;
  da.gate = gate;
  da.hist = at<int>(ws, L.hist);
  da.base = at<int>(ws, L.base);
  da.counts = counts;
  da.offsets = offsets;
  da.ucoff = at<int>(ws, L.ucoff);
  da.perm_token = perm_token;
  da.perm_slot = nullptr;
  da.row_of = row_of;
  da.gate_sorted = gate ? at<float>(ws, L.gate_sorted) : nullptr;
  if (plan_experts) {  // expert GEMM tile prefix and tile tables, when the experts follow
    da.seg_mblk = at<int>(ws, L.mprefix);
    da.mblk_rows = kExpertBM;
    da.tab1 = at<int4>(ws, L.tab1);
    da.tab2 = at<int4>(ws, L.tab2);
    da.nblk1 = (int)ceil_div(c.f, kExpertBN);
    da.nblk2 = (int)ceil_div(c.d, kExpertBN);
    da.mdone = at<int>(ws, L.mdone);
  }
  da.status = status;
  return launch_dispatch(da, st);
}

int run_experts(const moe_config &c, const Layout &L, const void *x_perm, const int *offsets,
                const moe_expert_params &ep, void *y_perm, void *ws, int *status,
                cudaStream_t st, int plan_ready = 0, const char *name = nullptr) {
  ExpertArgs e{};
  e.name = name;
  e.x_perm = x_perm;
  e.offsets = offsets;
  e.mprefix = at<int>(ws, L.mprefix);
  e.tab1 = at<int4>(ws, L.tab1);
  e.tab2 = at<int4>(ws, L.tab2);
  e.mdone = at<int>(ws, L.mdone);
  e.plan_ready = plan_ready;
  e.n = c.n;
  e.d = c.d;
  e.f = c.f;
  e.S = c.T * c.k;
  e.W1 = ep.W1;
  e.W2 = ep.W2;
  e.b1 = ep.b1;
  e.b2 = ep.b2;
  e.hid = at<void>(ws, L.hid);
  e.y_perm = y_perm;
  e.status = status;
  return c.expert_dtype == MOE_BF16 ? launch_expert_bf16(e, st) : launch_expert_f32(e, st);
}

bool gate_params_ok(const moe_config &c, const moe_gate_params *gp) {
  // the gate GEMM copies weight rows in 16-byte pieces
  if (!gp || !gp->W_g || !aligned(gp->W_g, 16)) return false;
  if (c.noise && (!gp->W_noise || !aligned(gp->W_noise, 16))) return false;
  if (c.hier_a > 0 && (!gp->W_g2 || !aligned(gp->W_g2, 16))) return false;
  if (c.hier_a > 0 && c.noise && (!gp->W_noise2 || !aligned(gp->W_noise2, 16))) return false;
  // the routing kernel reads the selection bias in 16-byte pieces
  if (c.router == MOE_ROUTER_SIGMOID && gp->sel_bias && !aligned(gp->sel_bias, 16)) return false;
  if (gp->seed_dev && !aligned(gp->seed_dev, 8)) return false;
  return true;
}

bool expert_params_ok(const moe_expert_params *ep) {
  return ep && ep->W1 && ep->W2 && aligned(ep->W1, 16) && aligned(ep->W2, 16);
}

bool shared_params_ok(const moe_config &c, const moe_expert_params *ep) {
  return !c.shared_expert ||
         (ep->W1s && ep->W2s && aligned(ep->W1s, 16) && aligned(ep->W2s, 16));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument or configuration";
    case MOE_EWORKSPACE: return "workspace too small or misaligned";
    case MOE_ECUDA: return "CUDA call or kernel launch failed";
    case MOE_EDEVICE: return "no usable sm_100 (B200) device";
    default: return "unknown error";
  }
}

int moe_validate(const moe_config *c) {
  if (!c) return MOE_EINVAL;
  if (c->gate_precision != MOE_GATE_FP32 && c->gate_precision != MOE_GATE_TF32X3) return MOE_EINVAL;
  if (c->T < 0 || c->n < 1 || c->n > 8192 || c->k < 1 || c->k > kMaxK || c->k > c->n)
    return MOE_EINVAL;
  if (c->d < 8 || c->d % 8 || c->d > 16384 || c->f < 8 || c->f % 8 || c->f > 65536)
    return MOE_EINVAL;
  if (c->router != MOE_ROUTER_NOISY_TOPK && c->router != MOE_ROUTER_SWITCH &&
      c->router != MOE_ROUTER_SIGMOID)
    return MOE_EINVAL;
  if (c->router == MOE_ROUTER_SIGMOID && (c->noise || c->hier_a)) return MOE_EINVAL;
  if (c->shared_expert != 0 && c->shared_expert != 1) return MOE_EINVAL;
  if (c->router_stats != 0 && c->router_stats != 1) return MOE_EINVAL;
  if (c->backward != 0 && c->backward != 1) return MOE_EINVAL;
  if (!(c->w_z == c->w_z) || !(c->w_entropy == c->w_entropy)) return MOE_EINVAL;  // NaN
  if (c->noise != 0 && c->noise != 1) return MOE_EINVAL;
  if (c->expert_dtype != MOE_F32 && c->expert_dtype != MOE_BF16) return MOE_EINVAL;
  if (c->overflow_passthrough != 0 && c->overflow_passthrough != 1) return MOE_EINVAL;
  if (!(c->capacity_factor == c->capacity_factor)) return MOE_EINVAL;  // NaN
  if (c->router == MOE_ROUTER_SWITCH && (c->k != 1 || c->noise || c->hier_a || c->n > 4096))
    return MOE_EINVAL;
  if (c->hier_a < 0) return MOE_EINVAL;
  if (c->hier_a > 0) {
    if (c->hier_b < 1 || (int64_t)c->hier_a * c->hier_b != c->n) return MOE_EINVAL;
    if (c->hier_k1 < 1 || c->hier_k1 > c->hier_a || c->hier_k1 > kMaxK) return MOE_EINVAL;
    if (c->hier_k2 < 1 || c->hier_k2 > c->hier_b || c->hier_k2 > kMaxK) return MOE_EINVAL;
    if (c->hier_k1 * c->hier_k2 != c->k) return MOE_EINVAL;
  }
  if ((int64_t)c->T * c->k > INT_MAX / 2) return MOE_EINVAL;
  if (c->token_base < 0 || c->token_base + (int64_t)c->T > (int64_t)1 << 32) return MOE_EINVAL;
  return MOE_OK;
}

int moe_capacity(const moe_config *cfg, int64_t *C) {
  const int v = moe_validate(cfg);
  if (v != MOE_OK) return v;
  if (!C) return MOE_EINVAL;
  *C = capacity_of(*cfg);
  return MOE_OK;
}

int moe_workspace_size(const moe_config *cfg, size_t *bytes) {
  const int v = moe_validate(cfg);
  if (v != MOE_OK) return v;
  if (!bytes) return MOE_EINVAL;
  *bytes = make_layout(*cfg).total;
  return MOE_OK;
}

int moe_gate(const moe_config *cfg, const float *x, const moe_gate_params *gp, int32_t *topk_idx,
             float *topk_gate, float *load, float *prob_sum, void *ws, size_t ws_bytes,
             int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  if (!load || !gate_params_ok(c, gp)) return MOE_EINVAL;
  if (c.T > 0 && (!x || !aligned(x, 16) || !topk_idx || !topk_gate)) return MOE_EINVAL;
  return run_gate(c, L, x, *gp, topk_idx, topk_gate, load, prob_sum, ws, status,
                  reinterpret_cast<cudaStream_t>(stream));
}

int moe_dispatch(const moe_config *cfg, const float *x, const int32_t *topk_idx, int32_t *counts,
                 int32_t *offsets, int32_t *perm_token, int32_t *row_of, void *x_perm, void *ws,
                 size_t ws_bytes, int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  if (!counts || !offsets) return MOE_EINVAL;
  if (c.T > 0 && (!topk_idx || !perm_token || !row_of)) return MOE_EINVAL;
  if (c.T > 0 && (x == nullptr) != (x_perm == nullptr)) return MOE_EINVAL;
  if (c.T > 0 && x && (!aligned(x, 16) || !aligned(x_perm, 16))) return MOE_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run_dispatch(c, L, topk_idx, nullptr, capacity_of(c), counts, offsets, perm_token,
                      row_of, x, x_perm, ws, status, st);
}

int moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                   const moe_expert_params *ep, void *y_perm, void *ws, size_t ws_bytes,
                   int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  if (!offsets || !expert_params_ok(ep)) return MOE_EINVAL;
  if (c.T > 0 && (!x_perm || !y_perm || !aligned(x_perm, 16) || !aligned(y_perm, 16)))
    return MOE_EINVAL;
  return run_experts(c, L, x_perm, offsets, *ep, y_perm, ws, status,
                     reinterpret_cast<cudaStream_t>(stream));
}

int moe_combine(const moe_config *cfg, const void *y_perm, const float *topk_gate,
                const int32_t *row_of, const float *x, float *y, int32_t *status,
                moe_stream_t stream) {
  const int v = moe_validate(cfg);
  if (v != MOE_OK) return v;
  const moe_config &c = *cfg;
  if (!status) return MOE_EINVAL;
  if (c.T > 0 && (!y_perm || !topk_gate || !row_of || !y || !aligned(y, 16) ||
                  !aligned(y_perm, 16)))
    return MOE_EINVAL;
  if (c.T > 0 && c.overflow_passthrough && (!x || !aligned(x, 16))) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_combine(y_perm, c.expert_dtype == MOE_BF16, topk_gate, row_of, x,
                        c.overflow_passthrough, c.T, c.k, c.d, y, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

int moe_balance_losses(const moe_config *cfg, const int32_t *topk_idx, const float *topk_gate,
                       const int32_t *counts, const float *load, const float *prob_sum,
                       float *importance, float *losses, void *ws, size_t ws_bytes,
                       int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  if (!counts || !load || !importance || !losses) return MOE_EINVAL;
  if (c.T > 0 && (!topk_idx || !topk_gate)) return MOE_EINVAL;
  if (c.router == MOE_ROUTER_SWITCH && !prob_sum) return MOE_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // gates sorted by expert (stable), from a capacity-free dispatch into scratch
  MOE_TRY(run_dispatch(c, L, topk_idx, topk_gate, INT64_MAX, at<int>(ws, L.counts_scratch),
                       at<int>(ws, L.offsets), at<int>(ws, L.perm_token), at<int>(ws, L.row_of),
                       nullptr, nullptr, ws, status, st));
  MOE_TRY(launch_importance(at<float>(ws, L.gate_sorted), at<int>(ws, L.ucoff), c.n, importance,
                            st));
  return launch_losses(importance, load, counts, prob_sum, c.n, c.T, c.k, capacity_of(c), c.router,
                       c.w_importance, c.w_load, c.alpha_aux, nullptr, losses, st);
}

int moe_forward(const moe_config *cfg, const float *x, const moe_gate_params *gp,
                const moe_expert_params *ep, float *y, int32_t *topk_idx, float *topk_gate,
                float *importance, float *load, int32_t *counts, float *losses, void *ws,
                size_t ws_bytes, int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  if (!importance || !load || !counts || !losses) return MOE_EINVAL;
  if (c.T > 0 && (!x || !y || !topk_idx || !topk_gate || !aligned(x, 16) || !aligned(y, 16)))
    return MOE_EINVAL;
  if (!gate_params_ok(c, gp) || !expert_params_ok(ep) || !shared_params_ok(c, ep))
    return MOE_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool sw = c.router == MOE_ROUTER_SWITCH;
  float *prob_sum = sw ? at<float>(ws, L.prob_sum) : nullptr;
  const int64_t C = capacity_of(c);
  int *offsets = at<int>(ws, L.offsets);
  int *row_of = at<int>(ws, L.row_of);
  void *x_perm = at<void>(ws, L.x_perm);
  void *y_perm = at<void>(ws, L.y_perm);

  Side *side = nullptr;
  MOE_TRY(side_stream(&side));
  MOE_TRY(run_gate(c, L, x, *gp, topk_idx, topk_gate, load, prob_sum, ws, status, st, side));
  const bool tc = c.expert_dtype == MOE_BF16;
  void *x_shared = c.shared_expert ? at<void>(ws, L.x_shared) : nullptr;
  void *y_shared = c.shared_expert ? at<void>(ws, L.y_shared) : nullptr;
  int *shared_off = c.shared_expert ? at<int>(ws, L.shared_off) : nullptr;
  MOE_TRY(run_dispatch(c, L, topk_idx, topk_gate, C, counts, offsets, at<int>(ws, L.perm_token),
                       row_of, x, x_perm, ws, status, st, tc, x_shared, shared_off));
  // balance statistics beside the expert chain; they read only the gate's and
  // the dispatch's outputs
  MOE_TRY(stream_after(side->s, st, side->fork_dispatch));
  MOE_TRY(launch_importance(at<float>(ws, L.gate_sorted), at<int>(ws, L.ucoff), c.n, importance,
                            side->s));
  MOE_TRY(launch_losses(importance, load, counts, prob_sum, c.n, c.T, c.k, C, c.router,
                        c.w_importance, c.w_load, c.alpha_aux,
                        c.router_stats ? at<float>(ws, L.rstats) : nullptr, losses, side->s));
  if (c.T > 0) {
    MOE_TRY(run_experts(c, L, x_perm, offsets, *ep, y_perm, ws, status, st, tc ? 1 : 0));
    if (c.shared_expert) {
      // every token through the shared expert: one expert, rows 0..T-1 in
      // token order, its plan written by the dispatch; the routed launch is
      // done with the hidden-layer rows by now, so they are reused
      ExpertArgs e{};
      e.name = tc ? "shared_expert_ffn_tcgen05" : "shared_expert_ffn_fp32";
      e.x_perm = x_shared;
      e.offsets = shared_off;
      e.mprefix = at<int>(ws, L.shared_mprefix);
      e.tab1 = at<int4>(ws, L.shared_tab1);
      e.tab2 = at<int4>(ws, L.shared_tab2);
      e.mdone = at<int>(ws, L.shared_mdone);
      e.plan_ready = 1;
      e.n = 1;
      e.d = c.d;
      e.f = c.f;
      e.S = c.T;
      e.W1 = ep->W1s;
      e.W2 = ep->W2s;
      e.b1 = ep->b1s;
      e.b2 = ep->b2s;
      // the backward pass needs both hidden layers: the shared one then has its own rows
      e.hid = at<void>(ws, c.backward ? L.hid_shared : L.hid);
      e.y_perm = y_shared;
      e.status = status;
      MOE_TRY(tc ? launch_expert_bf16(e, st) : launch_expert_f32(e, st));
    }
    MOE_TRY(launch_combine(y_perm, c.expert_dtype == MOE_BF16, topk_gate, row_of, x,
                           c.overflow_passthrough, c.T, c.k, c.d, y, y_shared, st));
  }
  return stream_after(st, side->s, side->join);
}

int moe_backward(const moe_config *cfg, const float *x, const moe_gate_params *gp,
                 const moe_expert_params *ep, const float *dy, const int32_t *topk_idx,
                 const float *topk_gate, const float *importance, const float *load,
                 const int32_t *counts, float *dx, const moe_grads *gr, void *ws,
                 size_t ws_bytes, int32_t *status, moe_stream_t stream) {
  Layout L;
  MOE_TRY(common_checks(cfg, ws, ws_bytes, status, &L));
  const moe_config &c = *cfg;
  const bool hier = c.hier_a > 0;
  if (!c.backward || (hier && c.shared_expert)) return MOE_EINVAL;
  if (!gr || !gr->dW1 || !gr->dW2 || !importance || !load || !counts) return MOE_EINVAL;
  if (!aligned(gr->dW1, 16) || !aligned(gr->dW2, 16)) return MOE_EINVAL;
  if (c.T > 0 && (!x || !dy || !dx || !topk_idx || !topk_gate || !aligned(x, 16) ||
                  !aligned(dy, 16) || !aligned(dx, 16)))
    return MOE_EINVAL;
  if (!gate_params_ok(c, gp) || !expert_params_ok(ep) || !shared_params_ok(c, ep))
    return MOE_EINVAL;
  if (c.shared_expert && (!gr->dW1s || !gr->dW2s || !aligned(gr->dW1s, 16) ||
                          !aligned(gr->dW2s, 16)))
    return MOE_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int T = c.T, d = c.d, n = c.n, k = c.k, f = c.f;
  const int ng = hier ? c.hier_a : n;  // width of the flat / primary gate
  const size_t S = (size_t)T * k;
  auto zero = [&](float *p, size_t cnt) -> int {
    if (!p || cnt == 0) return MOE_OK;
    return cudaMemsetAsync(p, 0, 4 * cnt, st) == cudaSuccess ? MOE_OK : MOE_ECUDA;
  };
  if (T == 0) {  // no tokens: every gradient is zero
    MOE_TRY(zero(gr->dW_g, (size_t)d * ng));
    MOE_TRY(zero(gr->db_g, ng));
    if (c.noise) MOE_TRY(zero(gr->dW_noise, (size_t)d * ng));
    if (hier) {
      const size_t ab = (size_t)c.hier_a * c.hier_b;
      MOE_TRY(zero(gr->dW_g2, ab * d));
      MOE_TRY(zero(gr->db_g2, ab));
      if (c.noise) MOE_TRY(zero(gr->dW_noise2, ab * d));
    }
    MOE_TRY(zero(gr->dW1, (size_t)n * f * d));
    MOE_TRY(zero(gr->db1, (size_t)n * f));
    MOE_TRY(zero(gr->dW2, (size_t)n * d * f));
    MOE_TRY(zero(gr->db2, (size_t)n * d));
    if (c.shared_expert) {
      MOE_TRY(zero(gr->dW1s, (size_t)f * d));
      MOE_TRY(zero(gr->db1s, f));
      MOE_TRY(zero(gr->dW2s, (size_t)d * f));
      MOE_TRY(zero(gr->db2s, d));
    }
    return MOE_OK;
  }
  const int *offsets = at<int>(ws, L.offsets);
  const int *row_of = at<int>(ws, L.row_of);
  void *dy_perm = at<void>(ws, L.dy_perm), *dhid = at<void>(ws, L.dhid);
  void *dx_perm = at<void>(ws, L.dx_perm);
  void *dy_sh = c.shared_expert ? at<void>(ws, L.dy_shared) : nullptr;
  void *dhid_sh = c.shared_expert ? at<void>(ws, L.dhid_shared) : nullptr;
  void *dx_sh = c.shared_expert ? at<void>(ws, L.dx_shared) : nullptr;
  float *dgate = at<float>(ws, L.dgate);
  float *lam_imp = at<float>(ws, L.lam_imp), *lam_load = at<float>(ws, L.lam_load);
  float *sw_coef = at<float>(ws, L.sw_coef);
  float *dc = at<float>(ws, L.dc), *dz = c.noise ? at<float>(ws, L.dz) : nullptr;

  // ---- balancing losses -> dL/dImportance, dL/dLoad, Switch dL/dp: one
  // block on the side stream, needed only by the gate's backward
  Side *side = nullptr;
  MOE_TRY(side_stream(&side));
  MOE_TRY(stream_after(side->s, st, side->fork_gate));
  MOE_TRY(launch_bwd_coef(importance, load, counts, n, T, c.w_importance, c.w_load, c.alpha_aux,
                          c.router, c.noise, lam_imp, lam_load, sw_coef, side->s));
  // ---- combine: dy_perm rows, dL/dgate, the shared expert's rows
  const bool tc = c.expert_dtype == MOE_BF16;
  MOE_TRY(launch_combine_bwd(dy, topk_gate, row_of, at<void>(ws, L.y_perm), tc, T, k, d, dy_perm,
                             dgate, dy_sh, st));
  if (!tc) {
    // fp32 experts: per expert, its rows in order, gradients accumulated in place
    MOE_TRY(launch_expert_bwd_f32(at<float>(ws, L.x_perm), static_cast<const float *>(dy_perm),
                                  offsets, n, d, f, static_cast<const float *>(ep->W1), ep->b1,
                                  static_cast<const float *>(ep->W2),
                                  static_cast<float *>(dx_perm), gr->dW1, gr->db1, gr->dW2,
                                  gr->db2, nullptr, st));
    if (c.shared_expert)
      MOE_TRY(launch_expert_bwd_f32(
          at<float>(ws, L.x_shared), static_cast<const float *>(dy_sh), at<int>(ws, L.shared_off),
          1, d, f, static_cast<const float *>(ep->W1s), ep->b1s,
          static_cast<const float *>(ep->W2s), static_cast<float *>(dx_sh), gr->dW1s, gr->db1s,
          gr->dW2s, gr->db2s, "shared_expert_bwd_fp32", st));
  } else {
  // ---- experts: dhid = (dy_perm W2) * [hid > 0], dx_perm = dhid W1 (the forward's tiles)
  const int64_t mb_upper = ceil_div((int64_t)S, kExpertBM) + n;
  if (cudaMemsetAsync(at<int>(ws, L.mdone), 0, 4 * (size_t)(mb_upper + 1), st) != cudaSuccess)
    return MOE_ECUDA;
  ExpertArgs e{};
  e.backward = 1;
  e.x_perm = dy_perm;
  e.offsets = offsets;
  e.mprefix = at<int>(ws, L.mprefix);
  e.tab1 = at<int4>(ws, L.tab1);
  e.tab2 = at<int4>(ws, L.tab2);
  e.mdone = at<int>(ws, L.mdone);
  e.plan_ready = 1;
  e.n = n;
  e.d = d;
  e.f = f;
  e.S = (int)S;
  e.W1 = ep->W1;
  e.W2 = ep->W2;
  e.hid = dhid;
  e.y_perm = dx_perm;
  e.mask = at<void>(ws, L.hid);
  e.status = status;
  MOE_TRY(launch_expert_bf16(e, st));
  WgradArgs w{};
  w.dy_perm = dy_perm;
  w.hid = at<void>(ws, L.hid);
  w.dhid = dhid;
  w.x_perm = at<void>(ws, L.x_perm);
  w.offsets = offsets;
  w.n = n;
  w.d = d;
  w.f = f;
  w.S = (int)S;
  w.dW1 = gr->dW1;
  w.dW2 = gr->dW2;
  w.status = status;
  MOE_TRY(launch_wgrad_bf16(w, st));
  MOE_TRY(launch_bias_grad(dy_perm, dhid, offsets, n, d, f, gr->db2, gr->db1, nullptr, st));
  if (c.shared_expert) {
    const int64_t mbe = ceil_div((int64_t)T, kExpertBM);
    if (cudaMemsetAsync(at<int>(ws, L.shared_mdone), 0, 4 * (size_t)(mbe + 1), st) != cudaSuccess)
      return MOE_ECUDA;
    ExpertArgs es = e;
    es.name = "shared_expert_bwd_tcgen05";
    es.x_perm = dy_sh;
    es.offsets = at<int>(ws, L.shared_off);
    es.mprefix = at<int>(ws, L.shared_mprefix);
    es.tab1 = at<int4>(ws, L.shared_tab1);
    es.tab2 = at<int4>(ws, L.shared_tab2);
    es.mdone = at<int>(ws, L.shared_mdone);
    es.n = 1;
    es.S = T;
    es.W1 = ep->W1s;
    es.W2 = ep->W2s;
    es.hid = dhid_sh;
    es.y_perm = dx_sh;
    es.mask = at<void>(ws, L.hid_shared);
    MOE_TRY(launch_expert_bf16(es, st));
    WgradArgs ws2 = w;
    ws2.name = "shared_wgrad_tcgen05";
    ws2.dy_perm = dy_sh;
    ws2.hid = at<void>(ws, L.hid_shared);
    ws2.dhid = dhid_sh;
    ws2.x_perm = at<void>(ws, L.x_shared);
    ws2.offsets = at<int>(ws, L.shared_off);
    ws2.n = 1;
    ws2.S = T;
    ws2.dW1 = gr->dW1s;
    ws2.dW2 = gr->dW2s;
    MOE_TRY(launch_wgrad_bf16(ws2, st));
    MOE_TRY(launch_bias_grad(dy_sh, dhid_sh, at<int>(ws, L.shared_off), 1, d, f, gr->db2s,
                             gr->db1s, "shared_bias_grad", st));
  }
  }  // bf16 experts
  // ---- dispatch: dx = sum of the token's expert rows (+ pass-through, + shared)
  MOE_TRY(launch_dx_gather(dx_perm, tc, row_of, dy, c.overflow_passthrough, T, k, d, dx_sh, dx,
                           st));
  // ---- gate: dL/dc, dL/dz per row, then the fp32 contractions
  GateBwdArgs g{};
  g.T = T;
  g.n = ng;
  g.k = k;
  g.c = at<float>(ws, L.c);
  g.s = at<float>(ws, L.s);
  g.idx = topk_idx;
  g.gate = topk_gate;
  g.dgate = dgate;
  g.lam_imp = lam_imp;
  g.lam_load = lam_load;
  g.sw_coef = sw_coef;
  g.kth = at<int4>(ws, L.kth);
  g.seed = c.seed;
  g.token_base = (uint32_t)c.token_base;
  g.seed_dev = reinterpret_cast<const unsigned long long *>(gp->seed_dev);
  g.router = c.router;
  g.noise = c.noise;
  g.has_load = c.noise && c.w_load != 0.f;
  g.dc = dc;
  g.dz = dz;
  MOE_TRY(stream_after(st, side->s, side->join));  // the loss coefficients
  if (hier) {
    // [SGMoE-note] "分层 MoE": the slot gradients split into the two levels,
    // the load coefficients too, then each level is a flat gate's backward
    const int a = c.hier_a, b = c.hier_b, k1 = c.hier_k1, k2 = c.hier_k2, R2 = T * k1;
    float *lam_p = at<float>(ws, L.lam_p), *lam_s = at<float>(ws, L.lam_s);
    float *dgp = at<float>(ws, L.dgp), *dgs = at<float>(ws, L.dgs);
    const int *grow = at<int>(ws, L.g_row_of);
    if (g.has_load)
      MOE_TRY(launch_hier_coef(lam_load, at<float>(ws, L.load_p), at<float>(ws, L.load2),
                               at<int>(ws, L.g_counts), a, b, lam_p, lam_s, st));
    MOE_TRY(launch_hier_split(T, k1, k2, k, n, at<float>(ws, L.pgate), grow,
                              topk_idx, dgate, at<float>(ws, L.gate2), lam_imp, dgp, dgs, st));
    g.k = k1;  // the primary gate over the groups
    g.idx = at<int>(ws, L.pidx);
    g.gate = at<float>(ws, L.pgate);
    g.dgate = dgp;
    g.lam_imp = nullptr;  // folded into dgp
    g.lam_load = lam_p;
    MOE_TRY(launch_gate_bwd(g, st));
    GateBwdArgs g2 = g;  // the secondary gates, one row per (token, kept group)
    g2.T = R2;
    g2.n = b;
    g2.k = k2;
    g2.c = at<float>(ws, L.c2);
    g2.s = at<float>(ws, L.s2);
    g2.idx = at<int>(ws, L.idx2);
    g2.gate = at<float>(ws, L.gate2);
    g2.dgate = dgs;
    g2.lam_load = lam_s;
    g2.kth = at<int4>(ws, L.kth2);
    g2.row_token = at<int>(ws, L.g_perm_token);
    g2.seg_off = at<int>(ws, L.g_offsets);
    g2.G = a;
    g2.dc = at<float>(ws, L.dc2);
    g2.dz = c.noise ? at<float>(ws, L.dz2) : nullptr;
    MOE_TRY(launch_gate_bwd(g2, st));
    MOE_TRY(launch_hier_gate_wgrad(x, d, g2.row_token, g2.seg_off, a, b, g2.dc, g2.dz, gr->dW_g2,
                                   c.noise ? gr->dW_noise2 : nullptr, gr->db_g2, st));
  } else {
    MOE_TRY(launch_gate_bwd(g, st));
  }
  if (c.w_z != 0.f || c.w_entropy != 0.f)  // router z-loss and gate entropy terms
    MOE_TRY(launch_gate_stats_bwd(at<float>(ws, L.c), T, ng, c.w_z, c.w_entropy, dc, st));
  if (gr->db_g) MOE_TRY(launch_colsum(dc, T, ng, at<float>(ws, L.colsum_part), gr->db_g, st));
  float *sp = at<float>(ws, L.sgemm_part);
  const bool want_n = c.noise && gr->dW_noise;
  // the split count the workspace was sized for (two problems with noise)
  const int splits = sgemm_splits(d, ng, T, c.noise ? 2 : 1);
  if (gr->dW_g || want_n) {
    // dW_g = x^T dc and dW_noise = x^T dz: M = d, N = ng, K = T, A shared
    SgemmArgs a{};
    a.M = d; a.N = ng; a.K = T;
    a.A[0] = a.A[1] = x; a.lda = d; a.at = 1;
    a.ldb = ng; a.bt = 0; a.ldc = ng;
    if (gr->dW_g && want_n) {
      a.B[0] = dc; a.C[0] = gr->dW_g;
      a.B[1] = dz; a.C[1] = gr->dW_noise;
      a.nprob = 2;
    } else {
      a.B[0] = gr->dW_g ? dc : dz;
      a.C[0] = gr->dW_g ? gr->dW_g : gr->dW_noise;
      a.nprob = 1;
    }
    a.part = splits > 1 ? sp : nullptr;
    a.splits = splits;
    a.name = "gate_wgrad_fp32";
    MOE_TRY(launch_sgemm(a, st));
  }
  {
    // dx += dc W_g^T (+ dz W_noise^T): M = T, N = d, K = ng; B(k, q) = W[q][k]
    SgemmArgs a{};
    a.M = T; a.N = d; a.K = ng;
    a.A[0] = dc; a.A[1] = dz; a.lda = ng; a.at = 0;
    a.B[0] = gp->W_g; a.B[1] = gp->W_noise; a.ldb = ng; a.bt = 1;
    a.C[0] = a.C[1] = dx; a.ldc = d;
    a.nprob = 1;
    a.ksum = c.noise ? 1 : 0;
    a.accumulate = 1;
    a.splits = 1;
    a.name = "gate_dgrad_fp32";
    MOE_TRY(launch_sgemm(a, st));
  }
  if (hier) {  // dx += the secondary gates' part, row by row, then per token in order
    const int a = c.hier_a, b = c.hier_b, k1 = c.hier_k1, R2 = T * k1;
    MOE_TRY(launch_hier_gate_dgrad(at<float>(ws, L.dc2), c.noise ? at<float>(ws, L.dz2) : nullptr,
                                   gp->W_g2, gp->W_noise2, at<int>(ws, L.g_offsets),
                                   at<int>(ws, L.g_mblk), (int)ceil_div(R2, kGateBM) + a, a, d, b,
                                   at<float>(ws, L.dxs), T, k1, at<int>(ws, L.g_row_of), dx, st));
  }
  if (gr->dgate &&
      cudaMemcpyAsync(gr->dgate, dgate, 4 * S, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ECUDA;
  if (!hier && gr->dlogits && cudaMemcpyAsync(gr->dlogits, dc, 4 * (size_t)T * n,
                                              cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ECUDA;
  return MOE_OK;
}

int moe_fma_probe(float *out, int blocks, int iters, int packed, moe_stream_t stream) {
  if (!out || blocks < 1 || iters < 1) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_fma_probe(out, blocks, iters, packed ? 1 : 0, reinterpret_cast<cudaStream_t>(stream));
}

int moe_gather_rows(const void *src, const int32_t *index, void *dst, int64_t rows,
                    int64_t row_bytes, int64_t src_rows, int32_t *status, moe_stream_t stream) {
  if (rows < 0 || src_rows < 0 || row_bytes <= 0 || row_bytes % 16) return MOE_EINVAL;
  if (rows > 0 && (!src || !index || !dst || !aligned(src, 16) || !aligned(dst, 16)))
    return MOE_EINVAL;
  if (!status) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_gather_rows(src, index, dst, rows, row_bytes, src_rows, status,
                            reinterpret_cast<cudaStream_t>(stream));
}

int moe_balance_from_totals(const moe_config *cfg, const float *importance, const float *load,
                            const int32_t *counts, const float *prob_sum, const float *dropped,
                            float *losses, int32_t *status, moe_stream_t stream) {
  MOE_TRY(moe_validate(cfg));
  const moe_config &c = *cfg;
  if (!importance || !load || !counts || !dropped || !losses || !status) return MOE_EINVAL;
  if (c.router == MOE_ROUTER_SWITCH && !prob_sum) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_losses(importance, load, counts, prob_sum, c.n, c.T, c.k, INT64_MAX, c.router,
                       c.w_importance, c.w_load, c.alpha_aux, nullptr, losses,
                       reinterpret_cast<cudaStream_t>(stream), dropped);
}

int moe_test_expert_wait(unsigned long long limit_ns, int withhold_mblock) {
  set_expert_wait(limit_ns, withhold_mblock);
  return MOE_OK;
}

int moe_noise_step(uint64_t *seed_dev, moe_stream_t stream) {
  if (!seed_dev || !aligned(seed_dev, 8)) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_noise_step(reinterpret_cast<unsigned long long *>(seed_dev),
                           reinterpret_cast<cudaStream_t>(stream));
}

int moe_sel_bias_update(const moe_config *cfg, const int32_t *counts, float gamma,
                        float *sel_bias, moe_stream_t stream) {
  MOE_TRY(moe_validate(cfg));
  if (!counts || !sel_bias) return MOE_EINVAL;
  MOE_TRY(check_device());
  return launch_sel_bias_update(counts, cfg->n, cfg->T, cfg->k, gamma, sel_bias,
                                reinterpret_cast<cudaStream_t>(stream));
}

int moe_trace_enable(int on) {
  g_trace = on != 0;
  return MOE_OK;
}

int moe_trace_reset(void) {
  trace_collect();
  g_agg.clear();
  return MOE_OK;
}

int moe_trace_count(void) {
  trace_collect();
  return (int)g_agg.size();
}

int moe_trace_get(int i, const char **name, int *launches, double *total_ms) {
  trace_collect();
  if (i < 0 || i >= (int)g_agg.size()) return MOE_EINVAL;
  if (name) *name = g_agg[i].name.c_str();
  if (launches) *launches = g_agg[i].launches;
  if (total_ms) *total_ms = g_agg[i].ms;
  return MOE_OK;
}

long long moe_launch_count(void) { return g_launches; }

}  // extern "C"
