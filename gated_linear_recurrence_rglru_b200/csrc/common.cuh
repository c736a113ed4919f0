// Shared device helpers of the RG-LRU kernels: storage-type conversion and the
// scalar pieces of the layer (softplus of -Lambda, sigmoid, log-space decay).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rglru.h"

namespace rglru {

constexpr float kDecayC = 8.0f;  // c in log a_t = -c * r_t * softplus(-Lambda)

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T> __device__ __forceinline__ float ldg_f32(const T *p) {
  return to_f32<T>(__ldg(p));
}

// softplus(v) = log(1 + e^v) without overflow or cancellation.
__device__ __forceinline__ float softplus_f32(float v) {
  return fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
}

__device__ __forceinline__ float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

// One element of the layer after the gate pre-activations are known:
// r = sigmoid(za), i = sigmoid(zx), log a = -c r sp, a = e^(log a),
// beta = sqrt(1 - a^2) * i * u with 1 - a^2 formed as -expm1(2 log a).
__device__ __forceinline__ void decay_and_input(float za, float zx, float u, float neg_c_sp,
                                                float &a, float &beta, float &log_a) {
  const float r = sigmoid_f32(za);
  const float i = sigmoid_f32(zx);
  log_a = neg_c_sp * r;
  a = expf(log_a);
  beta = sqrtf(-expm1f(2.0f * log_a)) * (i * u);
}

// GeLU(v) = v Phi(v) = v (1 + erf(v / sqrt 2)) / 2, the exact form (the gating
// of the recurrent block around the layer).
__device__ __forceinline__ float gelu_exact(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

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

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace rglru
