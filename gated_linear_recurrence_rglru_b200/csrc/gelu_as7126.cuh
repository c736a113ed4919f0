// GeLU of the recurrent block's tensor-core GEMM epilogue, with erf from a
// published rational-exponential approximation.
#pragma once

#include <cstdint>

namespace rglru {

// Coefficients of erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5)
// exp(-x^2) + e(x), t = 1 / (1 + p x), x >= 0, |e(x)| <= 1.5e-7: Abramowitz and
// Stegun, Handbook of Mathematical Functions, formula 7.1.26.
namespace erf_as7126 {
constexpr float kP = 0.3275911f;
constexpr float kA1 = 0.254829592f;
constexpr float kA2 = -0.284496736f;
constexpr float kA3 = 1.421413741f;
constexpr float kA4 = -1.453152027f;
constexpr float kA5 = 1.061405429f;
}  // namespace erf_as7126

// GeLU(v) = v Phi(v) with Phi(-|v|) = erfc(|v| / sqrt 2) / 2 from formula
// 7.1.26 above (one reciprocal and one base-2 exponential on the special
// function unit): |Phi error| <= 7.5e-8 plus the approximate reciprocal's and
// exponential's rounding, far below the bf16 rounding of the gated output.
// Phi(|v|) is taken as 1 - Phi(-|v|), so nothing cancels for negative v.
__device__ __forceinline__ float gelu_as7126(float v) {
  using namespace erf_as7126;
  const float x = fabsf(v) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(kP, x, 1.0f));
  const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, kA5, kA4), kA3), kA2), kA1);
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-x * x * 1.44269504088896341f));
  const float phi_neg = 0.5f * poly * e;
  return v * (v >= 0.0f ? 1.0f - phi_neg : phi_neg);
}

}  // namespace rglru
