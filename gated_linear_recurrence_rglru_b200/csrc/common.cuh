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

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace rglru
