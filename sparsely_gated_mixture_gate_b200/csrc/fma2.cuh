// fma2.cuh -- packed fp32 multiply-adds for the CUDA-core GEMMs.
//
// fma.rn.f32x2 computes two independent fp32 FMAs on the halves of 64-bit
// register pairs, each rounded once to nearest as fmaf would be, so a GEMM
// that keeps its accumulators in pairs produces bitwise the results of the
// scalar form while issuing half the FMA instructions.
#pragma once

namespace moe {

// two fp32 values as one 64-bit register pair, and back
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long p;
  asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(lo), "f"(hi));
  return p;
}
__device__ __forceinline__ void unpack2(unsigned long long p, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
// d = a * b + d on both halves
__device__ __forceinline__ void fma2(unsigned long long &d, unsigned long long a,
                                     unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

}  // namespace moe
