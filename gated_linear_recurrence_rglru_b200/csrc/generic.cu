// Generic RG-LRU kernels: fp32 arithmetic on CUDA cores for any I/O type.
//
// Forward over a sequence (the layer's definition, include/rglru.h; run as a
// linear scan, S. De's thread on Griffin):
// time is cut into nseg segments so that B * H * nseg blocks fill the GPU.
//   pass 1  aggregate: per (b, segment, channel) the segment's decay product
//           A = prod a_t and its local state H (scan from zero);
//   pass 2  carry: one thread per (b, channel) chains the (A, H) pairs in time
//           order, h_in(s+1) = A_s h_in(s) + H_s, starting from h0;
//   pass 3  final: each segment rescans from its h_in and writes y.
// With a single segment only pass 3 runs. Nothing waits on another block, so
// the path needs no device-side timeout.
//
// One block per (segment, head, batch row); thread j owns channel h*bw + j.
// Per group of TB tokens a block stages the Conv1D outputs of the whole head
// in shared memory, then every thread forms its two gate pre-activations with
// bw fused multiply-adds per token and gate.
#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

constexpr int kTB = 8;  // tokens per shared-memory stage

template <typename T>
__device__ __forceinline__ float hist_value(const T *xb, const T *cs_in_b, int t, int D, int d) {
  // x_t for t >= 0, else the chronological conv state (slot 3 + t), else zero.
  if (t >= 0) return ldg_f32(xb + (size_t)t * D + d);
  if (cs_in_b != nullptr) return ldg_f32(cs_in_b + (size_t)(3 + t) * D + d);
  return 0.0f;
}

template <typename T, bool kAggregate>
__global__ void __launch_bounds__(1024)
fwd_generic_kernel(FwdArgs p, int L, int nseg, float *__restrict__ ws_A,
                   float *__restrict__ ws_H, const float *__restrict__ ws_hin) {
  extern __shared__ float u_s[];  // [kTB][bw]
  const int bw = p.D / p.H;
  const int j = threadIdx.x;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const bool active = j < bw;
  const int D = p.D;
  const int d = h * bw + (active ? j : 0);
  const int t0 = s * L;
  const int t1 = min(p.T, t0 + L);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  const size_t seg_idx = ((size_t)b * nseg + s) * D + d;

  float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, ba = 0.f, bx = 0.f, neg_c_sp = 0.f;
  float xm3 = 0.f, xm2 = 0.f, xm1 = 0.f, hcur = 0.f, sum_la = 0.f;
  if (active) {
    const T *cw = static_cast<const T *>(p.conv_w);
    w0 = ldg_f32(cw + d);
    w1 = ldg_f32(cw + D + d);
    w2 = ldg_f32(cw + 2 * D + d);
    w3 = ldg_f32(cw + 3 * D + d);
    ba = ldg_f32(static_cast<const T *>(p.b_a) + d);
    bx = ldg_f32(static_cast<const T *>(p.b_x) + d);
    neg_c_sp = -kDecayC * softplus_f32(-__ldg(p.Lambda + d));
    xm3 = hist_value(xb, cs_in_b, t0 - 3, D, d);
    xm2 = hist_value(xb, cs_in_b, t0 - 2, D, d);
    xm1 = hist_value(xb, cs_in_b, t0 - 1, D, d);
    if (!kAggregate) {
      if (nseg > 1) hcur = ws_hin[seg_idx];
      else if (p.h0) hcur = p.h0[(size_t)b * D + d];
    }
  }
  T *yb = static_cast<T *>(p.y) + (size_t)b * p.T * D;

  for (int tb = t0; tb < t1; tb += kTB) {
    float u_own[kTB];
#pragma unroll
    for (int k = 0; k < kTB; ++k) {
      const int t = tb + k;
      float u = 0.f;
      if (active && t < t1) {
        const float xv = ldg_f32(xb + (size_t)t * D + d);
        u = fmaf(w3, xv, fmaf(w2, xm1, fmaf(w1, xm2, w0 * xm3)));
        xm3 = xm2;
        xm2 = xm1;
        xm1 = xv;
      }
      u_own[k] = u;
      if (active) u_s[k * bw + j] = u;
    }
    __syncthreads();
    if (active) {
      float za[kTB], zx[kTB];
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        za[k] = ba;
        zx[k] = bx;
      }
      for (int i = 0; i < bw; ++i) {
        const float wa = ldg_f32(Wa + (size_t)i * bw + j);
        const float wx = ldg_f32(Wx + (size_t)i * bw + j);
#pragma unroll
        for (int k = 0; k < kTB; ++k) {
          const float ui = u_s[k * bw + i];
          za[k] = fmaf(ui, wa, za[k]);
          zx[k] = fmaf(ui, wx, zx[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        const int t = tb + k;
        if (t < t1) {
          float a, beta, la;
          decay_and_input(za[k], zx[k], u_own[k], neg_c_sp, a, beta, la);
          hcur = fmaf(a, hcur, beta);
          sum_la += la;
          if (!kAggregate) yb[(size_t)t * D + d] = from_f32<T>(hcur);
        }
      }
    }
    __syncthreads();
  }

  if (!active) return;
  if (kAggregate) {
    ws_A[seg_idx] = expf(sum_la);
    ws_H[seg_idx] = hcur;
  } else if (s == nseg - 1) {
    if (p.h_T) p.h_T[(size_t)b * D + d] = hcur;
    if (p.conv_state_out) {
      T *cs = static_cast<T *>(p.conv_state_out) + (size_t)b * 3 * D;
      cs[d] = from_f32<T>(xm3);
      cs[D + d] = from_f32<T>(xm2);
      cs[2 * D + d] = from_f32<T>(xm1);
    }
  }
}

__global__ void carry_kernel(int B, int D, int nseg, const float *__restrict__ ws_A,
                             const float *__restrict__ ws_H, const float *__restrict__ h0,
                             float *__restrict__ ws_hin) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D) return;
  const int b = idx / D, d = idx - (idx / D) * D;
  float h = h0 ? h0[idx] : 0.f;
  for (int s = 0; s < nseg; ++s) {
    const size_t o = ((size_t)b * nseg + s) * D + d;
    ws_hin[o] = h;
    h = fmaf(ws_A[o], h, ws_H[o]);
  }
}

template <typename T>
__global__ void __launch_bounds__(1024) decode_generic_kernel(DecArgs p, int RB) {
  extern __shared__ float u_s[];  // [RB][bw]
  constexpr int kMaxRB = 8;
  const int bw = p.D / p.H;
  const int j = threadIdx.x;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * RB;
  const bool active = j < bw;
  const int D = p.D;
  const int d = h * bw + (active ? j : 0);
  const int s0 = p.pos % 3, s1 = (p.pos + 1) % 3, s2 = (p.pos + 2) % 3;
  float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, ba = 0.f, bx = 0.f, neg_c_sp = 0.f;
  if (active) {
    const T *cw = static_cast<const T *>(p.conv_w);
    w0 = ldg_f32(cw + d);
    w1 = ldg_f32(cw + D + d);
    w2 = ldg_f32(cw + 2 * D + d);
    w3 = ldg_f32(cw + 3 * D + d);
    ba = ldg_f32(static_cast<const T *>(p.b_a) + d);
    bx = ldg_f32(static_cast<const T *>(p.b_x) + d);
    neg_c_sp = -kDecayC * softplus_f32(-__ldg(p.Lambda + d));
  }
  const T *xt = static_cast<const T *>(p.x_t);
  T *ring = static_cast<T *>(p.conv_state);
  float u_own[kMaxRB], x_own[kMaxRB];
#pragma unroll
  for (int r = 0; r < kMaxRB; ++r) {
    const int b = row0 + r;
    float u = 0.f, xv = 0.f;
    if (r < RB && active && b < p.B) {
      const T *rb = ring + (size_t)b * 3 * D;
      xv = to_f32<T>(xt[(size_t)b * D + d]);
      u = fmaf(w3, xv,
               fmaf(w2, to_f32<T>(rb[(size_t)s2 * D + d]),
                    fmaf(w1, to_f32<T>(rb[(size_t)s1 * D + d]),
                         w0 * to_f32<T>(rb[(size_t)s0 * D + d]))));
    }
    u_own[r] = u;
    x_own[r] = xv;
    if (r < RB && active) u_s[r * bw + j] = u;
  }
  __syncthreads();
  if (!active) return;
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  float za[kMaxRB], zx[kMaxRB];
#pragma unroll
  for (int r = 0; r < kMaxRB; ++r) {
    za[r] = ba;
    zx[r] = bx;
  }
  for (int i = 0; i < bw; ++i) {
    const float wa = ldg_f32(Wa + (size_t)i * bw + j);
    const float wx = ldg_f32(Wx + (size_t)i * bw + j);
#pragma unroll
    for (int r = 0; r < kMaxRB; ++r) {
      if (r < RB) {
        const float ui = u_s[r * bw + i];
        za[r] = fmaf(ui, wa, za[r]);
        zx[r] = fmaf(ui, wx, zx[r]);
      }
    }
  }
  T *yt = static_cast<T *>(p.y_t);
#pragma unroll
  for (int r = 0; r < kMaxRB; ++r) {
    const int b = row0 + r;
    if (r < RB && b < p.B) {
      float a, beta, la;
      decay_and_input(za[r], zx[r], u_own[r], neg_c_sp, a, beta, la);
      const size_t o = (size_t)b * D + d;
      const float hn = fmaf(a, p.h[o], beta);
      p.h[o] = hn;
      yt[o] = from_f32<T>(hn);
      ring[(size_t)b * 3 * D + (size_t)s0 * D + d] = from_f32<T>(x_own[r]);
    }
  }
}

}  // namespace

// ------------------------------------------------------------------ host --

GenericPlan generic_plan(int B, int T, int H) {
  // Enough segments for about two blocks per SM of a 148-SM B200, but no
  // segment shorter than 16 tokens.
  constexpr int kTargetBlocks = 296, kMinSeg = 16;
  const long units = (long)B * H;
  int nseg = (int)((kTargetBlocks + units - 1) / units);
  const int max_seg = ceil_div(T, kMinSeg);
  if (nseg > max_seg) nseg = max_seg;
  if (nseg < 1) nseg = 1;
  GenericPlan pl;
  pl.L = ceil_div(T, nseg);
  pl.nseg = ceil_div(T, pl.L);
  return pl;
}

size_t generic_workspace_bytes(int B, int T, int D, int H) {
  const GenericPlan pl = generic_plan(B, T, H);
  if (pl.nseg <= 1) return 0;
  return align_up(3 * (size_t)B * pl.nseg * D * sizeof(float), 256);
}

template <typename T>
static cudaError_t launch_fwd_generic_t(const FwdArgs &p, void *ws, cudaStream_t st) {
  const int bw = p.D / p.H;
  const GenericPlan pl = generic_plan(p.B, p.T, p.H);
  const int threads = ceil_div(bw, 32) * 32;
  const size_t smem = (size_t)kTB * bw * sizeof(float);
  const dim3 grid(pl.nseg, p.H, p.B);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fwd_generic_kernel<T, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fwd_generic_kernel<T, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (pl.nseg == 1) {
    fwd_generic_kernel<T, false><<<grid, threads, smem, st>>>(p, pl.L, 1, nullptr, nullptr,
                                                              nullptr);
    return cudaGetLastError();
  }
  float *ws_A = static_cast<float *>(ws);
  const size_t n = (size_t)p.B * pl.nseg * p.D;
  float *ws_H = ws_A + n;
  float *ws_hin = ws_H + n;
  fwd_generic_kernel<T, true><<<grid, threads, smem, st>>>(p, pl.L, pl.nseg, ws_A, ws_H, nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int bd = p.B * p.D;
  carry_kernel<<<ceil_div(bd, 256), 256, 0, st>>>(p.B, p.D, pl.nseg, ws_A, ws_H, p.h0, ws_hin);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fwd_generic_kernel<T, false><<<grid, threads, smem, st>>>(p, pl.L, pl.nseg, nullptr, nullptr,
                                                            ws_hin);
  return cudaGetLastError();
}

cudaError_t launch_fwd_generic(const FwdArgs &p, int io, void *ws, cudaStream_t st) {
  cudaError_t e;
  if (p.ev_begin != nullptr && (e = cudaEventRecord(p.ev_begin, st)) != cudaSuccess) return e;
  e = io == RGLRU_IO_F32 ? launch_fwd_generic_t<float>(p, ws, st)
                         : launch_fwd_generic_t<__nv_bfloat16>(p, ws, st);
  if (e != cudaSuccess) return e;
  if (p.ev_end != nullptr) return cudaEventRecord(p.ev_end, st);
  return cudaSuccess;
}

int generic_kernel_launches(int B, int T, int H) {
  return generic_plan(B, T, H).nseg > 1 ? 3 : 1;
}

template <typename T>
static cudaError_t launch_decode_generic_t(const DecArgs &p, cudaStream_t st) {
  const int bw = p.D / p.H;
  const int RB = 8;
  const int threads = ceil_div(bw, 32) * 32;
  const size_t smem = (size_t)RB * bw * sizeof(float);
  const dim3 grid(ceil_div(p.B, RB), p.H);
  decode_generic_kernel<T><<<grid, threads, smem, st>>>(p, RB);
  return cudaGetLastError();
}

cudaError_t launch_decode_generic(const DecArgs &p, int io, cudaStream_t st) {
  if (io == RGLRU_IO_F32) return launch_decode_generic_t<float>(p, st);
  return launch_decode_generic_t<__nv_bfloat16>(p, st);
}

}  // namespace rglru
