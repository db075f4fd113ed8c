// gate_cutlass.cu -- the flat gate's two fp32 projections for wide gates
// (thousands of experts), on CUTLASS's SIMT GEMM templates:
//   c = x W_g + b_g            (epilogue: the bias row broadcast, ldc = 0)
//   s = Softplus(x W_noise)    (epilogue: Softplus of the accumulator)
// [SGMoE-xyz] "Noisy Top-K 門控"; fp32 multiply-adds throughout ([SGMoE-note]
// "缺点与局限性": the gate needs fp32).  Every output is the same fused
// multiply-add chain over k in order as in gate_gemm.cu's kernel, and the
// epilogues round as it does (bias added in one rounding; Softplus of the
// same formula), so the results are bitwise those of that kernel; for gates
// of 2048 or more columns per projection this mainloop (four-stage cp.async
// pipeline, 128 x 128 x 8 tiles, 32 x 64 warp tiles) runs about 17% faster
// (4096 experts: 49.9 against 42.7 TFLOP/s).  Non-finite values are caught by
// the routing kernel, which checks every H = c + eps * s.
#include "cutlass/cutlass.h"
#include "cutlass/epilogue/thread/activation.h"
#include "cutlass/epilogue/thread/linear_combination_generic.h"
#include "cutlass/gemm/device/gemm.h"

#include "internal.h"

namespace moe {
namespace {

template <typename T>
struct GateSoftplus {
  CUTLASS_HOST_DEVICE T operator()(T const &z) const {
    return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
  }
};
template <typename T, int N>
struct GateSoftplus<cutlass::Array<T, N>> {
  CUTLASS_HOST_DEVICE cutlass::Array<T, N> operator()(cutlass::Array<T, N> const &v) const {
    cutlass::Array<T, N> r;
    GateSoftplus<T> op;
    CUTLASS_PRAGMA_UNROLL
    for (int i = 0; i < N; ++i) r[i] = op(v[i]);
    return r;
  }
};

using RowMajor = cutlass::layout::RowMajor;
using ScaleType = cutlass::epilogue::thread::ScaleType;
template <template <typename> class Act, ScaleType::Kind Scale>
using Epilogue = cutlass::epilogue::thread::LinearCombinationGeneric<Act, float, 1, float, float, Scale>;
template <class Ep>
using SimtGemm = cutlass::gemm::device::Gemm<
    float, RowMajor, float, RowMajor, float, RowMajor, float, cutlass::arch::OpClassSimt,
    cutlass::arch::Sm80, cutlass::gemm::GemmShape<128, 128, 8>, cutlass::gemm::GemmShape<32, 64, 8>,
    cutlass::gemm::GemmShape<1, 1, 1>, Ep, cutlass::gemm::threadblock::GemmIdentityThreadblockSwizzle<>,
    4, 1, 1>;
using GemmBias =  // D = acc + bias row
    SimtGemm<Epilogue<cutlass::epilogue::thread::Identity, ScaleType::NoBetaScaling>>;
using GemmPlain = SimtGemm<Epilogue<cutlass::epilogue::thread::Identity, ScaleType::Nothing>>;  // D = acc
using GemmSoftplus = SimtGemm<Epilogue<GateSoftplus, ScaleType::Nothing>>;  // D = Softplus(acc)

template <class G>
int run(typename G::Arguments const &args, cudaStream_t st) {
  G gemm;
  if (gemm.can_implement(args) != cutlass::Status::kSuccess) return MOE_EINVAL;
  if (gemm.initialize(args, nullptr, st) != cutlass::Status::kSuccess) return MOE_ECUDA;
  int slot = -1;
  trace_begin("gate_gemm_fp32", st, &slot);
  const cutlass::Status s = gemm.run(st);
  const cudaError_t e = cudaGetLastError();
  trace_end(slot, st);
  count_launch();
  return (s == cutlass::Status::kSuccess && e == cudaSuccess) ? MOE_OK : MOE_ECUDA;
}

}  // namespace

bool gate_gemm_cutlass_applies(const GateGemmArgs &a) {
  return !a.seg_off && !a.row_token && a.nb >= kGateCutlassMinCols && a.R > 0;
}

int launch_gate_gemm_cutlass(const GateGemmArgs &a, cudaStream_t st) {
  const cutlass::gemm::GemmCoord size(a.R, a.nb, a.d);
  const cutlass::TensorRef<float const, RowMajor> x(a.x, a.d);
  if (a.bias) {
    // the bias row read for every output row: a source tensor of stride 0
    MOE_TRY(run<GemmBias>(GemmBias::Arguments(size, x, {a.Wg, a.nb}, {a.bias, 0}, {a.c, a.nb},
                                              {1.f, 1.f}),
                          st));
  } else {
    MOE_TRY(run<GemmPlain>(GemmPlain::Arguments(size, x, {a.Wg, a.nb}, {a.c, a.nb}, {a.c, a.nb},
                                                {1.f, 0.f}),
                           st));
  }
  if (a.noise)
    MOE_TRY(run<GemmSoftplus>(GemmSoftplus::Arguments(size, x, {a.Wn, a.nb}, {a.s, a.nb},
                                                      {a.s, a.nb}, {1.f, 0.f}),
                              st));
  return MOE_OK;
}

}  // namespace moe
