// dispatch_static.cu -- moe_dispatch_noalloc: the dispatch step with its
// scratch memory inside the library instead of in a caller workspace.
//
// Who needs it: callers that are handed only their input and output buffers
// and cannot obtain more device memory -- e.g. a plugin slot of a host
// inference engine that plans all memory up front and passes no allocator,
// or a serving loop that must not call cudaMalloc after start-up (the call
// synchronises the device and can fail under memory pressure).  For them the
// scratch of the dispatch (the per-block histograms, their scanned bases and
// the uncapped expert offsets) lives in one fixed array below.
//
// The array is a file-scope __device__ object, so every GPU that loads this
// library holds it (kScratchInts ints = 4 MiB) until the process exits.  Host
// code may not use the symbol as a pointer: its device address is looked up
// once per device with cudaGetSymbolAddress, with that device current, by the
// first call made on the device.  All calls share the array.  Each call
// writes every element it later reads (histograms, bases and offsets are
// fully rewritten), so nothing from an earlier call leaks into a result; two
// calls whose kernels overlap on the GPU (different streams, or different
// host threads on one stream without ordering) race on the array.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace moe {
namespace {

constexpr int64_t kScratchInts = MOE_DISPATCH_NOALLOC_SCRATCH_INTS;
static __device__ __align__(256) int g_dispatch_scratch[kScratchInts];

std::mutex g_mu;
int *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once).
int scratch_on_current_device(int **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_EDEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) return MOE_ECUDA;
    g_scratch_ptr[dev] = static_cast<int *>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_dispatch_noalloc(const moe_config *cfg, const float *x, const int32_t *topk_idx,
                                    int32_t *counts, int32_t *offsets, int32_t *perm_token,
                                    int32_t *row_of, void *x_perm, int32_t *status,
                                    moe_stream_t stream) {
  const int v = moe_validate(cfg);
  if (v != MOE_OK) return v;
  const moe_config &c = *cfg;
  if (!status || !counts || !offsets) return MOE_EINVAL;
  if (c.T > 0 && (!topk_idx || !perm_token || !row_of)) return MOE_EINVAL;
  if (c.T > 0 && (x == nullptr) != (x_perm == nullptr)) return MOE_EINVAL;
  auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (c.T > 0 && x && (!al16(x) || !al16(x_perm))) return MOE_EINVAL;

  // scratch: hist [B][n], base [B][n], uncapped offsets [n+1], the scan's ticket
  const int64_t B = ceil_div(c.T, dispatch_tokens_per_block(c.T));
  const int64_t need = 2 * B * (int64_t)c.n + c.n + 2;
  if (need > kScratchInts) return MOE_EWORKSPACE;  // beyond the fixed array

  // the device first: on anything but an sm_100 part the library's module has
  // no image, so the symbol lookup would fail with a CUDA error instead
  MOE_TRY(check_device());
  int *scratch = nullptr;
  MOE_TRY(scratch_on_current_device(&scratch));

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DispatchArgs da{};
  da.idx = topk_idx;
  da.T = c.T;
  da.k = c.k;
  da.n = c.n;
  da.C = c.capacity_factor > 0.0
             ? (int64_t)ceil((double)c.T * (double)c.k * c.capacity_factor / (double)c.n)
             : INT64_MAX;
  da.hist = scratch;
  da.base = scratch + B * c.n;
  da.ucoff = scratch + 2 * B * c.n;
  da.ticket = scratch + 2 * B * c.n + c.n + 1;
  da.x = x;
  da.x_perm = x_perm;
  da.d = c.d;
  da.x_bf16 = c.expert_dtype == MOE_BF16;
  da.counts = counts;
  da.offsets = offsets;
  da.perm_token = perm_token;
  da.row_of = row_of;
  da.status = status;
  return launch_dispatch(da, st);
}
