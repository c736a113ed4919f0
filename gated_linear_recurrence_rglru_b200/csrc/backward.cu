// Backward of the RG-LRU layer: the gradient of <dy, y> + <dh_T, h_T> with
// respect to every input ("Griffin: Mixing Gated Linear Recurrences with Local
// Attention for Efficient Language Models", section "Model Architecture"
// defines the forward; the backward is the chain rule through it, run as
// linear scans in both time directions, the forward's scheme in S. De's
// thread). fp32 arithmetic on CUDA cores for any I/O type.
//
// Time is cut into segments of at most kMaxSeg tokens; one block per
// (segment, head, batch row), thread j owning channel h*bw + j:
//   K1 aggregate  per segment: A = prod a_t, H = local state from zero and
//                 R = sum_t P_t dy_t with P_t = a_t0 ... a_t (the segment's
//                 contribution to the state gradient that leaves it leftwards);
//   K2 carry      per (b, channel): h_in of each segment in time order from h0,
//                 and C_s, the state gradient entering segment s from the right
//                 (dh_T for the last), in reverse order: C_{s-1} = R_s + A_s C_s,
//                 dh0 = R_0 + A_0 C_0;
//   K3 final      per segment: a forward sweep from h_in keeps the state at every
//                 8-token boundary in shared memory; a reverse sweep over the
//                 8-token groups recomputes each group (conv, gates), rebuilds
//                 h_{t-1}, runs G_t = dy_t + a_{t+1} G_{t+1} from C_s and forms
//                 d a = G h_{t-1}, d beta = G, g = sqrt(1 - a^2),
//                 d g = G i u, d i = G g u, d u = G g i + d z_a W_a^T + d z_x W_x^T,
//                 d la = d a a - d g a^2 / g, la = -c r sp, z -> r, i by sigmoid;
//                 it accumulates d b_a, d b_x and d Lambda per channel and writes
//                 u, d z_a, d z_x and d u to an fp32 workspace;
//   K4 weights    d W[h] = U_h^T dZ_h for both gates (32 x 32 tiles, the token
//                 sum split over blocks and combined with atomics);
//   K5 conv       d x_t = sum_k w[k] d u_{t+3-k} (t < 0: the conv history's
//                 gradient) and d w[k] = sum_t x_{t-3+k} d u_t.
// The path of d z_a through g carries r / g, which tends to 0 with r
// (1 - a^2 ~ 2 c sp r); it is formed as that ratio (0 where g = 0).
#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

constexpr int kTB = 8;         // tokens per group
constexpr int kMaxSeg = 512;   // tokens per segment: at most 64 boundary states per channel

template <typename T>
__device__ __forceinline__ float hist_x(const T *xb, const T *cs_in_b, int t, int D, int d) {
  if (t >= 0) return ldg_f32(xb + (size_t)t * D + d);
  if (cs_in_b != nullptr) return ldg_f32(cs_in_b + (size_t)(3 + t) * D + d);
  return 0.0f;
}

// Per-channel constants.
struct ChanC {
  float w0, w1, w2, w3, ba, bx, sp;
};

template <typename T>
__device__ __forceinline__ ChanC chan_c(const BwdArgs &p, int d) {
  const T *cw = static_cast<const T *>(p.conv_w);
  ChanC c;
  c.w0 = ldg_f32(cw + d);
  c.w1 = ldg_f32(cw + p.D + d);
  c.w2 = ldg_f32(cw + 2 * p.D + d);
  c.w3 = ldg_f32(cw + 3 * p.D + d);
  c.ba = ldg_f32(static_cast<const T *>(p.b_a) + d);
  c.bx = ldg_f32(static_cast<const T *>(p.b_x) + d);
  c.sp = softplus_f32(-__ldg(p.Lambda + d));
  return c;
}

// Gate weight (i, jj) of the head: from shared memory (fp32 rows of stride
// bw + 1, when kSW) or through L1 from global memory.
template <typename T, bool kSW>
__device__ __forceinline__ float w_at(const T *W, const float *Ws, int bw, int i, int jj) {
  return kSW ? Ws[i * (bw + 1) + jj] : ldg_f32(W + (size_t)i * bw + jj);
}

// Stages both gate weights of the head in shared memory, fp32, rows padded to
// bw + 1 floats: the gate contraction reads row i across the threads and the
// transposed one reads row j along a thread, both without bank conflicts.
template <typename T>
__device__ __forceinline__ void stage_weights(const T *Wa, const T *Wx, float *Wsa, float *Wsx,
                                              int bw) {
  for (int idx = threadIdx.x; idx < bw * bw; idx += blockDim.x) {
    const int i = idx / bw, jj = idx - (idx / bw) * bw;
    Wsa[i * (bw + 1) + jj] = ldg_f32(Wa + idx);
    Wsx[i * (bw + 1) + jj] = ldg_f32(Wx + idx);
  }
  __syncthreads();
}

// One group of kTB tokens from tb (own channel): Conv1D outputs u (the window
// xm3, xm2, xm1 = x_{tb-3..tb-1} advances), the head's u staged in u_s, then
// both gate pre-activations through the head's weights. Tokens at or past t1
// get u = 0 and are not used. Must be reached by every thread of the block.
template <typename T, bool kSW>
__device__ __forceinline__ void group_preacts(const T *xb, int D, int tb, int t1, int j, int bw,
                                              bool active, int d, const ChanC &c, float &xm3,
                                              float &xm2, float &xm1, float *u_s, const T *Wa,
                                              const T *Wx, const float *Wsa, const float *Wsx,
                                              float (&u)[kTB], float (&za)[kTB],
                                              float (&zx)[kTB]) {
#pragma unroll
  for (int k = 0; k < kTB; ++k) {
    const int t = tb + k;
    float uv = 0.f;
    if (active && t < t1) {
      const float xv = ldg_f32(xb + (size_t)t * D + d);
      uv = fmaf(c.w3, xv, fmaf(c.w2, xm1, fmaf(c.w1, xm2, c.w0 * xm3)));
      xm3 = xm2;
      xm2 = xm1;
      xm1 = xv;
    }
    u[k] = uv;
    if (active) u_s[k * bw + j] = uv;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kTB; ++k) {
    za[k] = c.ba;
    zx[k] = c.bx;
  }
  if (active) {
    for (int i = 0; i < bw; ++i) {
      const float wa = w_at<T, kSW>(Wa, Wsa, bw, i, j);
      const float wx = w_at<T, kSW>(Wx, Wsx, bw, i, j);
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        const float ui = u_s[k * bw + i];
        za[k] = fmaf(ui, wa, za[k]);
        zx[k] = fmaf(ui, wx, zx[k]);
      }
    }
  }
  __syncthreads();
}

template <typename T, bool kSW>
__global__ void __launch_bounds__(1024)
bwd_aggregate_kernel(BwdArgs p, int L, int nseg, float *__restrict__ ws_A,
                     float *__restrict__ ws_H, float *__restrict__ ws_R) {
  extern __shared__ float smem_a[];
  const int bw = p.D / p.H, D = p.D;
  float *u_s = smem_a;                            // [kTB][bw]
  float *Wsa = u_s + kTB * bw;                    // [bw][bw + 1] when kSW
  float *Wsx = Wsa + (kSW ? bw * (bw + 1) : 0);
  const int j = threadIdx.x;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const bool active = j < bw;
  const int d = h * bw + (active ? j : 0);
  const int t0 = s * L, t1 = min(p.T, t0 + L);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy) + (size_t)b * p.T * D;
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  if (kSW) stage_weights<T>(Wa, Wx, Wsa, Wsx, bw);
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float xm3 = 0.f, xm2 = 0.f, xm1 = 0.f;
  if (active) {
    c = chan_c<T>(p, d);
    xm3 = hist_x(xb, cs_in_b, t0 - 3, D, d);
    xm2 = hist_x(xb, cs_in_b, t0 - 2, D, d);
    xm1 = hist_x(xb, cs_in_b, t0 - 1, D, d);
  }
  const float neg_c_sp = -kDecayC * c.sp;
  float P = 1.f, Hl = 0.f, R = 0.f;
  for (int tb = t0; tb < t1; tb += kTB) {
    float u[kTB], za[kTB], zx[kTB];
    group_preacts<T, kSW>(xb, D, tb, t1, j, bw, active, d, c, xm3, xm2, xm1, u_s, Wa, Wx, Wsa,
                          Wsx, u, za, zx);
    if (active) {
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        const int t = tb + k;
        if (t < t1) {
          float a, beta, la;
          decay_and_input(za[k], zx[k], u[k], neg_c_sp, a, beta, la);
          Hl = fmaf(a, Hl, beta);
          P *= a;
          R = fmaf(P, ldg_f32(dyb + (size_t)t * D + d), R);
        }
      }
    }
  }
  if (!active) return;
  const size_t o = ((size_t)b * nseg + s) * D + d;
  ws_A[o] = P;
  ws_H[o] = Hl;
  ws_R[o] = R;
}

__global__ void bwd_carry_kernel(int B, int D, int nseg, const float *__restrict__ ws_A,
                                 const float *__restrict__ ws_H, const float *__restrict__ ws_R,
                                 const float *__restrict__ h0, const float *__restrict__ dh_T,
                                 float *__restrict__ ws_hin, float *__restrict__ ws_C,
                                 float *__restrict__ dh0) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D) return;
  const int b = idx / D, d = idx - (idx / D) * D;
  float hh = h0 ? h0[idx] : 0.f;
  for (int s = 0; s < nseg; ++s) {
    const size_t o = ((size_t)b * nseg + s) * D + d;
    ws_hin[o] = hh;
    hh = fmaf(ws_A[o], hh, ws_H[o]);
  }
  float cc = dh_T ? dh_T[idx] : 0.f;
  for (int s = nseg - 1; s >= 0; --s) {
    const size_t o = ((size_t)b * nseg + s) * D + d;
    ws_C[o] = cc;
    cc = fmaf(ws_A[o], cc, ws_R[o]);
  }
  if (dh0) dh0[idx] = cc;
}

template <typename T, bool kSW>
__global__ void __launch_bounds__(1024)
bwd_final_kernel(BwdArgs p, int L, int nseg, const float *__restrict__ ws_hin,
                 const float *__restrict__ ws_C, float *__restrict__ ws_u,
                 float *__restrict__ ws_dza, float *__restrict__ ws_dzx,
                 float *__restrict__ ws_du) {
  extern __shared__ float smem[];
  const int bw = p.D / p.H, D = p.D;
  float *u_s = smem;                    // [kTB][bw]
  float *dza_s = u_s + kTB * bw;        // [kTB][bw]
  float *dzx_s = dza_s + kTB * bw;      // [kTB][bw]
  float *Wsa = dzx_s + kTB * bw;        // [bw][bw + 1] when kSW
  float *Wsx = Wsa + (kSW ? bw * (bw + 1) : 0);
  float *hb_s = Wsx + (kSW ? bw * (bw + 1) : 0);   // [nsub][bw] state at each group start
  const int j = threadIdx.x;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const bool active = j < bw;
  const int d = h * bw + (active ? j : 0);
  const int t0 = s * L, t1 = min(p.T, t0 + L);
  const int nsub = (t1 - t0 + kTB - 1) / kTB;
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy) + (size_t)b * p.T * D;
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  const size_t seg = ((size_t)b * nseg + s) * D + d;
  if (kSW) stage_weights<T>(Wa, Wx, Wsa, Wsx, bw);
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (active) c = chan_c<T>(p, d);
  const float neg_c_sp = -kDecayC * c.sp;

  // ---- forward sweep: the state at every group start ----
  float xm3 = 0.f, xm2 = 0.f, xm1 = 0.f, hcur = 0.f;
  if (active) {
    xm3 = hist_x(xb, cs_in_b, t0 - 3, D, d);
    xm2 = hist_x(xb, cs_in_b, t0 - 2, D, d);
    xm1 = hist_x(xb, cs_in_b, t0 - 1, D, d);
    hcur = ws_hin[seg];
  }
  for (int g = 0; g < nsub; ++g) {
    const int tb = t0 + g * kTB;
    if (active) hb_s[g * bw + j] = hcur;
    float u[kTB], za[kTB], zx[kTB];
    group_preacts<T, kSW>(xb, D, tb, t1, j, bw, active, d, c, xm3, xm2, xm1, u_s, Wa, Wx, Wsa,
                          Wsx, u, za, zx);
    if (active) {
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        if (tb + k < t1) {
          float a, beta, la;
          decay_and_input(za[k], zx[k], u[k], neg_c_sp, a, beta, la);
          hcur = fmaf(a, hcur, beta);
        }
      }
    }
  }

  // ---- reverse sweep over the groups ----
  float gc = active ? ws_C[seg] : 0.f;   // a_{t+1} G_{t+1} for the token being processed
  float acc_sp = 0.f, acc_ba = 0.f, acc_bx = 0.f;
  const float csp = kDecayC * c.sp;
  for (int g = nsub - 1; g >= 0; --g) {
    const int tb = t0 + g * kTB;
    float w3 = 0.f, w2 = 0.f, w1 = 0.f;
    if (active) {
      w3 = hist_x(xb, cs_in_b, tb - 3, D, d);
      w2 = hist_x(xb, cs_in_b, tb - 2, D, d);
      w1 = hist_x(xb, cs_in_b, tb - 1, D, d);
    }
    float u[kTB], za[kTB], zx[kTB];
    group_preacts<T, kSW>(xb, D, tb, t1, j, bw, active, d, c, w3, w2, w1, u_s, Wa, Wx, Wsa, Wsx,
                          u, za, zx);
    float du_own[kTB];
    if (active) {
      float a[kTB], r[kTB], ig[kTB], gg[kTB], hp[kTB];
      float hh = hb_s[g * bw + j];
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        r[k] = sigmoid_f32(za[k]);
        ig[k] = sigmoid_f32(zx[k]);
        const float la = neg_c_sp * r[k];
        a[k] = expf(la);
        gg[k] = sqrtf(-expm1f(2.0f * la));
        hp[k] = hh;
        hh = fmaf(a[k], hh, gg[k] * ig[k] * u[k]);
      }
#pragma unroll
      for (int k = kTB - 1; k >= 0; --k) {
        const int t = tb + k;
        float dza = 0.f, dzx = 0.f, dub = 0.f;
        if (t < t1) {
          const float G = ldg_f32(dyb + (size_t)t * D + d) + gc;
          const float da = G * hp[k];
          const float dg = G * ig[k] * u[k];
          const float di = G * gg[k] * u[k];
          dub = G * gg[k] * ig[k];
          const float rog = gg[k] > 0.f ? r[k] / gg[k] : 0.f;
          const float aa = a[k] * a[k];
          dza = -csp * da * a[k] * r[k] * (1.f - r[k]) + csp * aa * (1.f - r[k]) * dg * rog;
          acc_sp += -kDecayC * da * a[k] * r[k] + kDecayC * aa * dg * rog;
          dzx = di * ig[k] * (1.f - ig[k]);
          acc_ba += dza;
          acc_bx += dzx;
          gc = a[k] * G;
          const size_t o = ((size_t)b * p.T + t) * D + d;
          ws_u[o] = u[k];
          ws_dza[o] = dza;
          ws_dzx[o] = dzx;
        }
        dza_s[k * bw + j] = dza;
        dzx_s[k * bw + j] = dzx;
        du_own[k] = dub;
      }
    }
    __syncthreads();
    if (active) {
      // d u_j += sum_m d z_a[m] W_a[j, m] + d z_x[m] W_x[j, m]
      float acc[kTB];
#pragma unroll
      for (int k = 0; k < kTB; ++k) acc[k] = du_own[k];
      for (int m = 0; m < bw; ++m) {
        const float wa = w_at<T, kSW>(Wa, Wsa, bw, j, m);
        const float wx = w_at<T, kSW>(Wx, Wsx, bw, j, m);
#pragma unroll
        for (int k = 0; k < kTB; ++k)
          acc[k] = fmaf(dza_s[k * bw + m], wa, fmaf(dzx_s[k * bw + m], wx, acc[k]));
      }
#pragma unroll
      for (int k = 0; k < kTB; ++k)
        if (tb + k < t1) ws_du[((size_t)b * p.T + tb + k) * D + d] = acc[k];
    }
    __syncthreads();
  }
  if (!active) return;
  atomicAdd(p.dLambda + d, acc_sp * (-sigmoid_f32(-__ldg(p.Lambda + d))));
  atomicAdd(p.db_a + d, acc_ba);
  atomicAdd(p.db_x + d, acc_bx);
}

// d W[h, i, j] += sum_n U[n, h bw + i] dZ[n, h bw + j] over one chunk of
// tokens; a 32 x 32 tile of (i, j) per block, 8 rows of threads.
__global__ void __launch_bounds__(256)
bwd_dw_kernel(const float *__restrict__ U, const float *__restrict__ dZa,
              const float *__restrict__ dZx, float *__restrict__ dWa, float *__restrict__ dWx,
              int N, int D, int H, int chunk) {
  __shared__ float us[32][33];
  __shared__ float zs[32][33];
  const int bw = D / H;
  const int tiles = (bw + 31) / 32;
  int tile = blockIdx.x;
  const int gate = tile % 2;
  tile /= 2;
  const int ti = tile % tiles, tj = (tile / tiles) % tiles, h = tile / (tiles * tiles);
  const float *Z = gate == 0 ? dZa : dZx;
  float *dW = gate == 0 ? dWa : dWx;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  const int i0 = ti * 32, j0 = tj * 32;
  const int n_begin = blockIdx.y * chunk, n_end = min(N, n_begin + chunk);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int n0 = n_begin; n0 < n_end; n0 += 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = n0 + ty + 8 * q;
      const bool ok = n < n_end;
      us[ty + 8 * q][tx] =
          ok && i0 + tx < bw ? U[(size_t)n * D + h * bw + i0 + tx] : 0.f;
      zs[ty + 8 * q][tx] =
          ok && j0 + tx < bw ? Z[(size_t)n * D + h * bw + j0 + tx] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int nn = 0; nn < 32; ++nn) {
      const float z = zs[nn][tx];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fmaf(us[nn][ty + 8 * q], z, acc[q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty + 8 * q, jj = j0 + tx;
    if (i < bw && jj < bw) atomicAdd(dW + ((size_t)h * bw + i) * bw + jj, acc[q]);
  }
}

// d x (and the conv history's gradient) from d u, and d w per channel for one
// chunk of tokens of one batch row; thread per channel.
template <typename T>
__global__ void bwd_conv_kernel(BwdArgs p, const float *__restrict__ du, int chunk) {
  const int D = p.D;
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (d >= D) return;
  const int m_begin = blockIdx.z * chunk, m_end = min(p.T + 3, m_begin + chunk);
  const T *cw = static_cast<const T *>(p.conv_w);
  float w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = ldg_f32(cw + (size_t)k * D + d);
  const float *dub = du + (size_t)b * p.T * D;
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  T *dxb = static_cast<T *>(p.dx) + (size_t)b * p.T * D;
  float dw[4] = {0.f, 0.f, 0.f, 0.f};
  // extended index m: x_{m-3}; d xe[m] = sum_k w[k] d u[m - k]; d w[k] += xe[m] d u[m - k]
  for (int m = m_begin; m < m_end; ++m) {
    const float xv = hist_x(xb, cs_in_b, m - 3, D, d);
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = m - k;
      if (t >= 0 && t < p.T) {
        const float g = dub[(size_t)t * D + d];
        acc = fmaf(w[k], g, acc);
        dw[k] = fmaf(xv, g, dw[k]);
      }
    }
    if (m >= 3) dxb[(size_t)(m - 3) * D + d] = from_f32<T>(acc);
    else if (p.dconv_state_in) p.dconv_state_in[((size_t)b * 3 + m) * D + d] = acc;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) atomicAdd(p.dconv_w + (size_t)k * D + d, dw[k]);
}

struct BwdPlan {
  int L, nseg;
};

BwdPlan bwd_plan(int B, int T, int H) {
  constexpr int kTargetBlocks = 296, kMinSeg = 16;
  const long units = (long)B * H;
  int nseg = (int)((kTargetBlocks + units - 1) / units);
  const int max_seg = ceil_div(T, kMinSeg);
  if (nseg > max_seg) nseg = max_seg;
  if (nseg < ceil_div(T, kMaxSeg)) nseg = ceil_div(T, kMaxSeg);
  if (nseg < 1) nseg = 1;
  BwdPlan pl;
  pl.L = ceil_div(T, nseg);
  pl.nseg = ceil_div(T, pl.L);
  return pl;
}

struct BwdLayout {
  size_t off_A, off_H, off_R, off_hin, off_C, off_u, off_dza, off_dzx, off_du, total;
};

BwdLayout bwd_layout(int B, int T, int D, int H) {
  const BwdPlan pl = bwd_plan(B, T, H);
  const size_t seg = align_up((size_t)B * pl.nseg * D * sizeof(float), 256);
  const size_t tok = align_up((size_t)B * T * D * sizeof(float), 256);
  BwdLayout L{};
  L.off_A = 0;
  L.off_H = L.off_A + seg;
  L.off_R = L.off_H + seg;
  L.off_hin = L.off_R + seg;
  L.off_C = L.off_hin + seg;
  L.off_u = L.off_C + seg;
  L.off_dza = L.off_u + tok;
  L.off_dzx = L.off_dza + tok;
  L.off_du = L.off_dzx + tok;
  L.total = L.off_du + tok;
  return L;
}

template <typename T, bool kSW>
cudaError_t launch_bwd_t(const BwdArgs &p, void *ws, cudaStream_t st) {
  const int bw = p.D / p.H;
  const BwdPlan pl = bwd_plan(p.B, p.T, p.H);
  const BwdLayout Ly = bwd_layout(p.B, p.T, p.D, p.H);
  unsigned char *w = static_cast<unsigned char *>(ws);
  float *A = reinterpret_cast<float *>(w + Ly.off_A), *Hh = reinterpret_cast<float *>(w + Ly.off_H);
  float *R = reinterpret_cast<float *>(w + Ly.off_R), *hin = reinterpret_cast<float *>(w + Ly.off_hin);
  float *C = reinterpret_cast<float *>(w + Ly.off_C), *U = reinterpret_cast<float *>(w + Ly.off_u);
  float *dza = reinterpret_cast<float *>(w + Ly.off_dza);
  float *dzx = reinterpret_cast<float *>(w + Ly.off_dzx);
  float *du = reinterpret_cast<float *>(w + Ly.off_du);
  const size_t D = p.D;
  cudaError_t e;
  // the accumulated gradients start at zero
  if ((e = cudaMemsetAsync(p.dconv_w, 0, 4 * D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dW_a, 0, D * bw * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dW_x, 0, D * bw * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.db_a, 0, D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.db_x, 0, D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dLambda, 0, D * sizeof(float), st)) != cudaSuccess) return e;

  const int threads = ceil_div(bw, 32) * 32;
  const dim3 grid(pl.nseg, p.H, p.B);
  const size_t wsm = kSW ? 2 * (size_t)bw * (bw + 1) * sizeof(float) : 0;
  const size_t smem1 = (size_t)kTB * bw * sizeof(float) + wsm;
  const int nsub_max = ceil_div(pl.L, kTB);
  const size_t smem3 = (size_t)(3 * kTB + nsub_max) * bw * sizeof(float) + wsm;
  if (smem1 > 48 * 1024 &&
      (e = cudaFuncSetAttribute(bwd_aggregate_kernel<T, kSW>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) !=
          cudaSuccess)
    return e;
  if (smem3 > 48 * 1024 &&
      (e = cudaFuncSetAttribute(bwd_final_kernel<T, kSW>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3)) !=
          cudaSuccess)
    return e;
  bwd_aggregate_kernel<T, kSW><<<grid, threads, smem1, st>>>(p, pl.L, pl.nseg, A, Hh, R);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int bd = p.B * p.D;
  bwd_carry_kernel<<<ceil_div(bd, 256), 256, 0, st>>>(p.B, p.D, pl.nseg, A, Hh, R, p.h0, p.dh_T,
                                                      hin, C, p.dh0);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_final_kernel<T, kSW><<<grid, threads, smem3, st>>>(p, pl.L, pl.nseg, hin, C, U, dza, dzx,
                                                          du);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int N = p.B * p.T;
  const int tiles = ceil_div(bw, 32);
  const int chunk = 1024;
  bwd_dw_kernel<<<dim3(2 * tiles * tiles * p.H, ceil_div(N, chunk)), dim3(32, 8), 0, st>>>(
      U, dza, dzx, p.dW_a, p.dW_x, N, p.D, p.H, chunk);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int cchunk = 256;
  bwd_conv_kernel<T><<<dim3(ceil_div(p.D, 128), p.B, ceil_div(p.T + 3, cchunk)), 128, 0, st>>>(
      p, du, cchunk);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int D, int H) { return bwd_layout(B, T, D, H).total; }

int bwd_launches() { return 5; }

cudaError_t launch_bwd(const BwdArgs &p, int io, void *ws, cudaStream_t st) {
  // both gate weights in shared memory (fp32) up to 128-wide heads: 2 x 129 x 128 x 4 B
  const bool sw = p.D / p.H <= 128;
  if (io == RGLRU_IO_F32)
    return sw ? launch_bwd_t<float, true>(p, ws, st) : launch_bwd_t<float, false>(p, ws, st);
  return sw ? launch_bwd_t<__nv_bfloat16, true>(p, ws, st)
            : launch_bwd_t<__nv_bfloat16, false>(p, ws, st);
}

}  // namespace rglru
