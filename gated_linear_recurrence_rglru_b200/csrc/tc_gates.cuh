// Device helpers shared by the tensor-core kernels: fast gate math of the
// RG-LRU (the layer's definition, include/rglru.h: r = sigmoid(z_a),
// i = sigmoid(z_x), log a = -c r softplus(-Lambda), beta = sqrt(1 - a^2) i u;
// gates that never read the state, "Beyond Transformer Architecture: Griffin
// and Google RecurrentGemma", "Core Components of Griffin", 1. RG-LRU),
// bf16 packing, and global-memory acquire/release accesses.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace rglru {
namespace gates {

constexpr float kLog2e = 1.4426950408889634f;
// Polynomials on w in [-1/8, 0], least-squares fits in relative error made for
// these kernels (constant terms pinned to 1):
//   e^w                         ~= 1 + w (E1 + w (E2 + w (E3 + w E4)))   max rel. error 1.3e-9
//   sqrt((1 - e^(2w)) / (-2w))  ~= 1 + w (G1 + w G2)                    max rel. error 8.0e-6
constexpr float kE1 = 0.99999986f, kE2 = 0.49998943f, kE3 = 0.16641409f, kE4 = 0.03923329f;
constexpr float kG1 = 0.49961998f, kG2 = 0.19817025f;
constexpr float kFastLimit = 0.125f;          // fast path when c * softplus(-Lambda) <= 1/8

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int *p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 64-bit single-copy-atomic accesses at GPU scope: a word written this way is
// read either whole or not at all, so a word that carries its own status needs
// no separate flag and no release/acquire fence.
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

// bf16 pair (low half = first element) -> two floats
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 v) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// Per-channel constants of the epilogue.
struct ChanK {
  float kba;    // -(b_a) log2 e
  float hbx;    // b_x / 2
  float nc;     // -c softplus(-Lambda): ln a_t = nc * r_t
  float nc2;    // nc log2 e (general path)
  // fast path, polynomials in r (ln a = nc r folded into the coefficients):
  //   a          = 1 + r (a1 + r (a2 + r (a3 + r a4))),  a_k = nc^k E_k
  //   2 sqrt(sp) sqrt(g(ln a)) = s0 + r (g1 + r g2),      g_k = s0 nc^k G_k
  float a1, a2, a3, a4;
  float s0, g1, g2;
};

// Fast path, two elements of one channel, valid when |nc| <= 1/8:
//   e = 2^(-(za + ba) log2 e), sqrt_r = (1 + e)^(-1/2), r = sqrt_r^2,
//   ln a = nc r, a = e^(ln a) (the polynomial above, in r),
//   sqrt(1 - a^2) = sqrt(-2 ln a) sqrt(g(ln a)) = 4 sqrt(sp) sqrt_r sqrt(g),
//   2 i = 1 + tanh((zx + bx) / 2),
//   beta = sqrt(1 - a^2) i u = sqrt_r * (2 sqrt(sp) sqrt(g)) * (u (1 + tanh)).
__device__ __forceinline__ void gate_pair_fast(float2 za, float2 zx, float2 u, const ChanK &k,
                                               float2 &a, float2 &beta) {
  const float2 earg = __ffma2_rn(za, f2(-kLog2e), f2(k.kba));
  float2 d = make_float2(ex2_approx(earg.x), ex2_approx(earg.y));
  d = __fadd2_rn(d, f2(1.0f));
  const float2 q = make_float2(rsqrt_approx(d.x), rsqrt_approx(d.y));
  const float2 r = __fmul2_rn(q, q);
  float2 pa = __ffma2_rn(r, f2(k.a4), f2(k.a3));
  pa = __ffma2_rn(r, pa, f2(k.a2));
  pa = __ffma2_rn(r, pa, f2(k.a1));
  a = __ffma2_rn(r, pa, f2(1.0f));
  float2 sg = __ffma2_rn(r, f2(k.g2), f2(k.g1));
  sg = __ffma2_rn(r, sg, f2(k.s0));                           // 2 sqrt(sp) sqrt(g)
  const float2 targ = __ffma2_rn(zx, f2(0.5f), f2(k.hbx));
  const float2 t = make_float2(tanh_approx(targ.x), tanh_approx(targ.y));
  const float2 tu = __ffma2_rn(t, u, u);                      // 2 i u
  beta = __fmul2_rn(__fmul2_rn(q, sg), tu);
}

// General path, one element: as above but a = 2^(log2 a) on the MUFU and
// 1 - a^2 = -expm1(2 ln a) by its series near a = 1, else 1 - a*a.
__device__ __forceinline__ void gate_one(float za, float zx, float u, const ChanK &k, float &a,
                                         float &beta, float &la) {
  const float e = ex2_approx(fmaf(za, -kLog2e, k.kba));
  const float q = rsqrt_approx(1.0f + e);
  const float r = q * q;
  const float ig = fmaf(0.5f, tanh_approx(fmaf(zx, 0.5f, k.hbx)), 0.5f);
  const float la2 = k.nc2 * r;
  la = k.nc * r;
  a = ex2_approx(la2);
  const float v = 2.0f * la;
  float p = fmaf(v, 1.0f / 720.0f, 1.0f / 120.0f);
  p = fmaf(v, p, 1.0f / 24.0f);
  p = fmaf(v, p, 1.0f / 6.0f);
  p = fmaf(v, p, 0.5f);
  p = fmaf(v, p, 1.0f);
  const float om = (v > -0.25f) ? (-v * p) : fmaf(-a, a, 1.0f);
  beta = sqrt_approx(om) * ig * u;
}


// Per-channel constants from the channel's bias pair and Lambda.
__device__ __forceinline__ ChanK chan_consts(float b_a, float b_x, float Lambda) {
  const float sp = softplus_f32(-Lambda);
  ChanK k;
  k.kba = -b_a * kLog2e;
  k.hbx = 0.5f * b_x;
  k.nc = -kDecayC * sp;
  k.nc2 = k.nc * kLog2e;
  const float n1 = k.nc, n2 = n1 * n1, n3 = n2 * n1, n4 = n2 * n2;
  k.a1 = n1 * kE1;
  k.a2 = n2 * kE2;
  k.a3 = n3 * kE3;
  k.a4 = n4 * kE4;
  k.s0 = 2.0f * sqrtf(sp);
  k.g1 = k.s0 * kG1 * n1;
  k.g2 = k.s0 * kG2 * n2;
  return k;
}

// True when the fast path is valid for this channel (c * softplus(-Lambda) <= 1/8).
__device__ __forceinline__ bool chan_fast(const ChanK &k) { return -k.nc <= kFastLimit; }

}  // namespace gates
}  // namespace rglru
