// fma_probe.cu -- a measurement helper beside the layer: a loop of
// independent fp32 fused multiply-adds that keeps every FP32 lane busy, so
// the host can time the GPU's FP32 FMA throughput with CUDA events.  That
// throughput is the roofline of the fp32 gate GEMM (the pages keep the gate
// in fp32, [SGMoE-note] "缺点与局限性"); measuring it replaces a figure
// derived from unit counts and clocks.
//
// Each thread runs CH independent chains v = v * m + a for iters x 8 steps
// (256 threads per block).  The packed form issues fma.rn.f32x2, two fp32
// FMAs per instruction on pairs of registers, so the two forms tell apart
// the FMA pipe's width and the issue rate.
#include "internal.h"

namespace moe {
namespace {

constexpr int CH = 16;  // independent chains per thread (scalar form)

__global__ void __launch_bounds__(256) fma_probe_scalar(float *out, int iters, float m, float a) {
  float v[CH];
#pragma unroll
  for (int j = 0; j < CH; ++j) v[j] = (float)(threadIdx.x + j) * 1e-3f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < CH; ++j) v[j] = fmaf(v[j], m, a);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < CH; ++j) s += v[j];
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__global__ void __launch_bounds__(256) fma_probe_packed(float *out, int iters, float m, float a) {
  unsigned long long v[CH / 2];
  const unsigned long long mm = pack2(m, m), aa = pack2(a, a);
#pragma unroll
  for (int j = 0; j < CH / 2; ++j)
    v[j] = pack2((float)(threadIdx.x + 2 * j) * 1e-3f, (float)(threadIdx.x + 2 * j + 1) * 1e-3f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < CH / 2; ++j)
        asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(v[j]) : "l"(mm), "l"(aa));
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < CH / 2; ++j) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v[j]));
    s += lo + hi;
  }
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

int launch_fma_probe(float *out, int blocks, int iters, int packed, cudaStream_t st) {
  const float m = 0.999f, a = 1e-3f;  // v stays bounded (fixed point 1)
  if (packed)
    return launch("fma_probe_f32x2", fma_probe_packed, dim3((unsigned)blocks), dim3(256), 0, st,
                  out, iters, m, a);
  return launch("fma_probe", fma_probe_scalar, dim3((unsigned)blocks), dim3(256), 0, st, out,
                iters, m, a);
}

}  // namespace moe
