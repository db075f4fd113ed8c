// ep.cu -- the row movement of the expert-parallel layer.
//
// [MoE-deep] §7.1: with the experts spread over devices, every token's rows
// travel to the device of their expert and the results travel back (two
// all-to-all exchanges per layer).  The exchanges deliver rows grouped by
// source rank; the expert kernel wants them grouped by expert.  This gather
// regroups them (and, with the inverse index, puts the results back in the
// exchange's order): dst row i = src row index[i], 16 bytes per thread and
// load, one warp per row, so every row moves as whole 128-byte segments.
#include "internal.h"

namespace moe {
namespace {

constexpr int NT = 256;

__global__ void __launch_bounds__(NT) gather_rows_kernel(const uint4 *__restrict__ src,
                                                         const int *__restrict__ index,
                                                         uint4 *__restrict__ dst, int64_t rows,
                                                         int q, int64_t src_rows, int *status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (NT / 32);
  bool bad = false;
  for (int64_t r = (int64_t)blockIdx.x * (NT / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int s = __ldg(index + r);
    const bool ok = s >= 0 && (int64_t)s < src_rows;
    bad |= !ok;
    const uint4 *from = src + (int64_t)(ok ? s : 0) * q;
    uint4 *to = dst + r * q;
    for (int c = lane; c < q; c += 32) to[c] = ok ? __ldg(from + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (bad && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_INDEX);
}

}  // namespace

int launch_gather_rows(const void *src, const int *index, void *dst, int64_t rows,
                       int64_t row_bytes, int64_t src_rows, int *status, cudaStream_t st) {
  if (rows == 0) return MOE_OK;
  const int q = (int)(row_bytes / 16);
  const int64_t blocks = ceil_div(rows, NT / 32);
  const int grid = (int)(blocks < 8 * (int64_t)num_sms() ? blocks : 8 * (int64_t)num_sms());
  return launch("gather_rows", gather_rows_kernel, dim3(grid), dim3(NT), 0, st,
                static_cast<const uint4 *>(src), index, static_cast<uint4 *>(dst), rows, q,
                src_rows, status);
}

}  // namespace moe
