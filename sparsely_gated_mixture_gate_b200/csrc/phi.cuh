// phi.cuh -- the standard normal CDF Phi of the smoothed load
// ([SGMoE-xyz] "負載平衡損失": P(x,i) = Phi((c_i - kth_excluding) / s_i)).
//
// For x = |z|, Phi(-x) = exp(-x^2/2) * Q(x), Q(x) = erfcx(x / sqrt 2) / 2.  Q
// is a degree-8 polynomial in t = 1 / (1 + 0.4 x) fitted on [0, 13.5] to
// relative error 7e-8 (phi_coef.py prints the coefficients and the error);
// x^2 is split into hi + lo exactly (one fma) so that exp(-x^2/2) keeps its
// relative accuracy in the tail.  Phi(z) = 1 - Phi(-z) for z > 0.  Largest
// relative error against Phi on [-12.5, 8]: 4.3e-7 (3.6 ulp); Phi(z) = 0
// below -13.5 (the exact value is below the smallest normal float there) and
// NaN stays NaN.  No branches: every lane of a warp runs the same instructions.
#pragma once

namespace moe {

__device__ __forceinline__ float phi_cdf(float z) {
  const float x = fabsf(z);
  const float t = __fdividef(1.0f, fmaf(0.4f, x, 1.0f));
  float q = -4.000047222e-02f;
  q = fmaf(q, t, 2.023256421e-01f);
  q = fmaf(q, t, -3.768121600e-01f);
  q = fmaf(q, t, 2.540788949e-01f);
  q = fmaf(q, t, -1.422286965e-02f);
  q = fmaf(q, t, 1.590774953e-01f);
  q = fmaf(q, t, 1.556458175e-01f);
  q = fmaf(q, t, 1.599203944e-01f);
  q = fmaf(q, t, -1.275824798e-05f);
  const float hi = x * x;
  const float lo = fmaf(x, x, -hi);
  const float e = expf(-0.5f * hi) * fmaf(-0.5f, lo, 1.0f);
  const float v = x >= 13.5f ? 0.0f : e * q;  // NaN falls through to e * q
  return z > 0.0f ? 1.0f - v : v;
}

}  // namespace moe
