// Backward of the RG-LRU layer: the gradient of <dy, y> + <dh_T, h_T> with
// respect to every input (the forward is the layer's definition stated in
// include/rglru.h; the backward is the chain rule through it, run as
// linear scans in both time directions, the forward's scheme in S. De's
// thread). fp32 arithmetic, except that for bf16 I/O with heads 32, 64 or
// 128 wide the two in-loop gate contractions (z = u W in K1, d z W^T in K3),
// and d W = U^T dZ for heads 64 or 128 wide, run on the tensor cores
// (warp-level bf16 MMA with fp32 accumulation, operands rounded to bf16 like
// the forward's u); fp32 I/O keeps them on CUDA cores.
//
// Time is cut into segments of L tokens (L a multiple of the 8-token group);
// a block holds S segments of one head and batch row, thread (sl, j) owning
// channel h*bw + j of segment sl, with the head's gate weights loaded once
// per block for all of them (fp32 rows in shared memory for the CUDA-core
// contractions; MMA fragments in registers in K1, bf16 rows in shared memory
// in K3 for the tensor-core ones):
//   K1 gates      per segment, in time order: Conv1D u, both gate
//                 pre-activations and gates (r, i -> fp32 workspace), the local scan
//                 from zero, whose (prod a, state) at each group start also go
//                 to the workspace, and the aggregates A = prod a_t,
//                 H = local end state and R = sum_t P_t dy_t with
//                 P_t = a_t0 ... a_t (the segment's contribution to the state
//                 gradient that leaves it leftwards);
//   K2 carry      per (b, channel), as a two-level scan over parts of the
//                 segments: h_in of each segment in time order from h0,
//                 and C_s, the state gradient entering segment s from the right
//                 (dh_T for the last), in reverse order: C_{s-1} = R_s + A_s C_s,
//                 dh0 = R_0 + A_0 C_0;
//   K3 final      per segment, groups in reverse order: the group's start state
//                 (prod a) h_in + (local state) and its stored r, i give
//                 h_{t-1}, a and beta for its 8 tokens; then G_t = dy_t +
//                 a_{t+1} G_{t+1} from C_s and d a = G h_{t-1}, d beta = G,
//                 g = sqrt(1 - a^2), d g = G i u, d i = G g u,
//                 d u = G g i + d z_a W_a^T + d z_x W_x^T,
//                 d la = d a a - d g a^2 / g, la = -c r sp, d z from r, i;
//                 it accumulates d b_a, d b_x and d Lambda per channel and writes
//                 u, d z_a, d z_x (over r, i; bf16 for the tensor-core d W) and
//                 d u to the workspace;
//   K4 weights    d W[h] = U_h^T dZ_h for both gates (64 x 64 tiles, the token
//                 sum split over blocks and combined with atomics; tensor cores
//                 or 4 x 4 FFMA tiles per thread);
//   K5 conv       d x_t = sum_k w[k] d u_{t+3-k} (t < 0: the conv history's
//                 gradient) and d w[k] = sum_t x_{t-3+k} d u_t.
// The path of d z_a through g carries r / g, which tends to 0 with r
// (1 - a^2 ~ 2 c sp r); it is formed as that ratio (0 where g = 0).
//
// Loads reach the arithmetic through shared memory, copied by cp.async ahead
// of use, so that no warp waits on a global load in its inner loop:
//   K1 (tensor-core version): the x and dy rows of each segment's group, a
//      ring of three slots filled two groups ahead;
//   K3 (tensor-core version): r, i, dy, the x rows of the Conv1D recompute and
//      the group-start pair, double-buffered one group ahead;
//   K4 (tensor-core version): U and d Z rows, a three-stage ring of 64-token
//      steps;
//   K5: each thread's own d u and x pairs, a private two-batch ring (no block
//      barrier: no thread reads another's slots).
// The CUDA-core versions of K1 and K3 issue L1 prefetches of the next group.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

constexpr int kTB = 8;       // tokens per group
constexpr int kRow = 12;     // floats per (channel, group) row in shared memory: 8 tokens and
                             // 4 pad, so 8 consecutive rows start on distinct 16-byte bank groups
constexpr int kMinSeg = 32;  // shortest segment the plan makes (unless T is shorter)
// threads the plan aims for: about four waves of 1024 threads on 148 SMs (any
// SM count works; the figure only sets the segment length)
constexpr long kTargetThreads = 4L * 148 * 1024;

struct BwdPlan {
  int L;      // tokens per segment, a multiple of kTB (the last segment may be shorter)
  int nseg;   // segments per sequence
  int S;      // segments per block
  int bwp;    // threads per segment: bw rounded up to a warp
};

BwdPlan bwd_plan(int B, int T, int D, int H) {
  const int bw = D / H;
  BwdPlan pl;
  pl.bwp = ceil_div(bw, 32) * 32;
  pl.S = (bw <= 64 ? 256 : 512) / pl.bwp;
  if (pl.S < 1) pl.S = 1;
  const long chans = (long)B * D;
  long nseg = (kTargetThreads + chans - 1) / chans;
  const long max_seg = ceil_div(T, kMinSeg);
  if (nseg > max_seg) nseg = max_seg;
  if (nseg < 1) nseg = 1;
  pl.L = ceil_div(ceil_div(T, (int)nseg), kTB) * kTB;
  pl.nseg = ceil_div(T, pl.L);
  return pl;
}

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

// Conv1D outputs of channel d for the group of kTB tokens from tb; tokens at
// or past t1 give 0.
template <typename T>
__device__ __forceinline__ void conv_group(const T *xb, const T *cs_in_b, int D, int d, int tb,
                                           int t1, const ChanC &c, float (&u)[kTB]) {
  float xm3 = hist_x(xb, cs_in_b, tb - 3, D, d);
  float xm2 = hist_x(xb, cs_in_b, tb - 2, D, d);
  float xm1 = hist_x(xb, cs_in_b, tb - 1, D, d);
#pragma unroll
  for (int k = 0; k < kTB; ++k) {
    const int t = tb + k;
    const float xv = t < t1 ? ldg_f32(xb + (size_t)t * D + d) : 0.f;
    u[k] = t < t1 ? fmaf(c.w3, xv, fmaf(c.w2, xm1, fmaf(c.w1, xm2, c.w0 * xm3))) : 0.f;
    xm3 = xm2;
    xm2 = xm1;
    xm1 = xv;
  }
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

__device__ __forceinline__ void store_row(float *row, const float (&v)[kTB]) {
  reinterpret_cast<float4 *>(row)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4 *>(row)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// One (segment, channel) thread of a block. Threads of segments past the end,
// and the pad threads of a head narrower than its warps, are inactive but
// take every barrier.
struct BwdThread {
  int sl, j, s, d, t0, t1;
  bool active;
};

__device__ __forceinline__ BwdThread bwd_thread(const BwdArgs &p, const BwdPlan &pl, int bw) {
  BwdThread th;
  th.sl = threadIdx.x / pl.bwp;
  th.j = threadIdx.x - th.sl * pl.bwp;
  th.s = blockIdx.x * pl.S + th.sl;
  th.t0 = min(p.T, th.s * pl.L);
  th.t1 = min(p.T, th.t0 + pl.L);
  th.active = th.j < bw && th.t0 < th.t1;
  th.d = blockIdx.y * bw + (th.j < bw ? th.j : 0);
  return th;
}

// ---- warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulate) ----
// Fragment layouts (PTX ISA, mma.m16n8k16 with .bf16): lane l, g = l / 4,
// q = l % 4. A (16 x 16, row-major): a0 = (g, 2q..2q+1), a1 = (g + 8, 2q..),
// a2 = (g, 2q + 8..), a3 = (g + 8, 2q + 8..). B (16 x 8): b0 = (k = 2q..2q+1,
// n = g), b1 = (k = 2q + 8.., n = g). C (16 x 8): c0, c1 = (g, 2q), (g, 2q + 1);
// c2, c3 = (g + 8, 2q), (g + 8, 2q + 1). Each pair holds the lower k (column)
// in its low half.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t shared_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16(unsigned short lo, unsigned short hi) {
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Geometry of the tensor-core kernels for a head width kBW in {32, 64, 128}:
// S segments of kBW threads per block, the block's M = 8 S tokens of a group
// as MT m-tiles of 16, kBW / 8 n-tiles of 8 channels, kBW / 16 k-steps. Warp w
// owns n-tile 2w / MT and the m-tiles 2w % MT and the next one.
template <int kBW>
struct TcGeo {
  static constexpr int kThreads = kBW == 128 ? 512 : 256;
  static constexpr int S = kThreads / kBW;
  static constexpr int M = S * kTB;
  static constexpr int MT = M / 16;
  static constexpr int NKS = kBW / 16;
  static constexpr int kStride = kBW + 8;   // bf16 per A row: 16-byte rows on distinct bank groups
  static_assert(MT % 2 == 0 && MT * (kBW / 8) == 2 * (kThreads / 32), "two tiles per warp");
};

// Brings the line holding p into L1 ahead of its load (a hint: no result, no fault).
__device__ __forceinline__ void prefetch_l1(const void *p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// 16-byte asynchronous global -> shared copy (zero-filled when !full: nothing is
// read from src then, which must still be a valid address); completed by
// cp_async_wait_all on the issuing thread, published to the block by a barrier.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool full) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(shared_addr(dst)),
               "l"(src), "r"(full ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// all but this thread's most recently committed group complete
__device__ __forceinline__ void cp_async_wait_one_pending() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Gate math of the backward in fp32 with about 1e-6 relative error: sigmoid
// and exp through the hardware base-2 exponential, approximate reciprocal and
// reciprocal square root; 1 - a^2 = -expm1(2 log a) by its Taylor series
// -x (1 + x/2 + x^2/6 + ... + x^6/5040) for |x| < 0.5 (truncation below 3e-7
// relative) and as 1 - e^x beyond (no cancellation there).
__device__ __forceinline__ float sigmoid_fast(float z) {
  return __fdividef(1.0f, 1.0f + __expf(-z));
}

__device__ __forceinline__ float neg_expm1_fast(float x) {   // x <= 0
  float p = fmaf(x, 1.f / 5040.f, 1.f / 720.f);
  p = fmaf(x, p, 1.f / 120.f);
  p = fmaf(x, p, 1.f / 24.f);
  p = fmaf(x, p, 1.f / 6.f);
  p = fmaf(x, p, 0.5f);
  p = fmaf(x, p, 1.0f);
  return x > -0.5f ? -x * p : 1.0f - __expf(x);
}

// r, i, a = e^(log a), g = sqrt(1 - a^2) and r / g (0 where g = 0) of one token.
struct TokGates {
  float r, i, a, g, rog;
};

// The same from the gates r = sigmoid(z_a) and i = sigmoid(z_x) themselves.
__device__ __forceinline__ TokGates tok_gates_ri(float r, float i, float neg_c_sp) {
  TokGates t;
  t.r = r;
  t.i = i;
  const float la = neg_c_sp * t.r;
  t.a = __expf(la);
  const float om = neg_expm1_fast(2.0f * la);
  const float rs = om > 0.f ? rsqrtf(om) : 0.f;
  t.g = om * rs;
  t.rog = t.r * rs;
  return t;
}

__device__ __forceinline__ TokGates tok_gates(float za, float zx, float neg_c_sp) {
  return tok_gates_ri(sigmoid_fast(za), sigmoid_fast(zx), neg_c_sp);
}

// The post-contraction part of a K1 group: decay, input, the local scan and
// the running R; the gates r and i of the live tokens to the workspace (K3
// needs z_a and z_x only through them). sdy: the
// group's dy rows staged in shared memory (this thread's channel at token 0,
// rows sstride apart), or nullptr to read dy from global memory.
template <typename T>
__device__ __forceinline__ void gates_scan_group(const float (&za)[kTB], const float (&zx)[kTB],
                                                 const float (&u)[kTB], int tb, int t1,
                                                 float neg_c_sp, const T *dyb, size_t orow,
                                                 int D, float &P, float &Hl, float &R,
                                                 float *__restrict__ ws_ga,
                                                 float *__restrict__ ws_gx,
                                                 const T *sdy = nullptr, int sstride = 0) {
#pragma unroll
  for (int k = 0; k < kTB; ++k) {
    const int t = tb + k;
    if (t < t1) {
      const TokGates q = tok_gates(za[k], zx[k], neg_c_sp);
      Hl = fmaf(q.a, Hl, q.g * (q.i * u[k]));
      P *= q.a;
      const size_t o = orow + (size_t)t * D;
      R = fmaf(P, sdy != nullptr ? to_f32<T>(sdy[k * sstride]) : ldg_f32(dyb + o), R);
      ws_ga[o] = q.r;
      ws_gx[o] = q.i;
    }
  }
}

template <typename T, bool kSW, int kMaxT>
__global__ void __launch_bounds__(kMaxT, kMaxT == 256 ? 3 : 1)
bwd_gates_kernel(BwdArgs p, BwdPlan pl, float *__restrict__ ws_A, float *__restrict__ ws_H,
                 float *__restrict__ ws_R, float *__restrict__ ws_gP, float *__restrict__ ws_gH,
                 float *__restrict__ ws_ga, float *__restrict__ ws_gx) {
  extern __shared__ float4 smem_g[];
  const int bw = p.D / p.H, D = p.D, h = blockIdx.y, b = blockIdx.z;
  const int seg_floats = pl.S * bw * kRow;
  float *u_s = reinterpret_cast<float *>(smem_g);   // [2][S][bw][kRow], double-buffered
  float *Wsa = u_s + 2 * seg_floats;                // [bw][bw + 1] when kSW
  float *Wsx = Wsa + (kSW ? bw * (bw + 1) : 0);
  const BwdThread th = bwd_thread(p, pl, bw);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy);
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  if (kSW) stage_weights<T>(Wa, Wx, Wsa, Wsx, bw);
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (th.active) c = chan_c<T>(p, th.d);
  const float neg_c_sp = -kDecayC * c.sp;
  const int ngt = ceil_div(p.T, kTB);
  const int jr = th.j < bw ? th.j : 0;
  const size_t orow = (size_t)b * p.T * D + th.d;
  float P = 1.f, Hl = 0.f, R = 0.f;
  const int ng = pl.L / kTB;
  for (int g = 0; g < ng; ++g) {
    const int tb = th.t0 + g * kTB;
    const bool live = th.active && tb < th.t1;
    const float *useg = u_s + (g & 1) * seg_floats + th.sl * bw * kRow;
    float u[kTB];
    if (live) {
      const size_t go = ((size_t)b * ngt + tb / kTB) * D + th.d;
      ws_gP[go] = P;
      ws_gH[go] = Hl;
      conv_group<T>(xb, cs_in_b, D, th.d, tb, th.t1, c, u);
    } else {
#pragma unroll
      for (int k = 0; k < kTB; ++k) u[k] = 0.f;
    }
    if (th.j < bw) store_row(const_cast<float *>(useg) + jr * kRow, u);
    __syncthreads();
    if (live) {
      float za[kTB], zx[kTB];
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        za[k] = c.ba;
        zx[k] = c.bx;
      }
      // z_j = b_j + sum_i u_i W[i, j]: the 8 tokens of u_i in two 16-byte reads
#pragma unroll 8
      for (int i = 0; i < bw; ++i) {
        const float4 u0 = reinterpret_cast<const float4 *>(useg + i * kRow)[0];
        const float4 u1 = reinterpret_cast<const float4 *>(useg + i * kRow)[1];
        const float wa = w_at<T, kSW>(Wa, Wsa, bw, i, th.j);
        const float wx = w_at<T, kSW>(Wx, Wsx, bw, i, th.j);
        const float uv[kTB] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int k = 0; k < kTB; ++k) {
          za[k] = fmaf(uv[k], wa, za[k]);
          zx[k] = fmaf(uv[k], wx, zx[k]);
        }
      }
      gates_scan_group<T>(za, zx, u, tb, th.t1, neg_c_sp, dyb, orow, D, P, Hl, R, ws_ga, ws_gx);
    }
  }
  if (!th.active) return;
  const size_t o = ((size_t)b * pl.nseg + th.s) * D + th.d;
  ws_A[o] = P;
  ws_H[o] = Hl;
  ws_R[o] = R;
}

// K1 for bf16 I/O and kBW in {32, 64, 128}: the gate contraction of each group
// on the tensor cores. u goes to shared memory as bf16 rows (token-major), each
// warp multiplies its two 16-token m-tiles by its 8 columns of W_a and W_x
// (fragments held in registers for the whole kernel), scatters the fp32
// results into (segment, channel) rows, and each thread reads back its own
// channel's 8 tokens for the scan. The x and dy rows of a group arrive in
// shared memory by cp.async two groups ahead of use.
template <int kBW>
__global__ void __launch_bounds__(TcGeo<kBW>::kThreads, kBW == 128 ? 1 : 3)
bwd_gates_tc_kernel(BwdArgs p, BwdPlan pl, float *__restrict__ ws_A, float *__restrict__ ws_H,
                    float *__restrict__ ws_R, float *__restrict__ ws_gP,
                    float *__restrict__ ws_gH, float *__restrict__ ws_ga,
                    float *__restrict__ ws_gx) {
  using T = __nv_bfloat16;
  using G = TcGeo<kBW>;
  extern __shared__ float4 smem_gt[];
  float *z_s = reinterpret_cast<float *>(smem_gt);                        // [S][2][kBW][kRow]
  T *u_s = reinterpret_cast<T *>(z_s + G::S * 2 * kBW * kRow);            // [M][kStride]
  // x rows tb-3 .. tb+7 and dy rows tb .. tb+7 of each segment's group, a ring of
  // three slots filled two groups ahead: [3][S][kTB + 3][kBW], [3][S][kTB][kBW]
  constexpr int XR = kTB + 3;
  T *xs_st = u_s + G::M * G::kStride;
  T *dys_st = xs_st + 3 * G::S * XR * kBW;
  const int D = p.D, h = blockIdx.y, b = blockIdx.z;
  const BwdThread th = bwd_thread(p, pl, kBW);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nt = (2 * warp) / G::MT, mt0 = (2 * warp) % G::MT;
  const int fg = lane >> 2, fq = lane & 3;
  // B[k = i][n = j] = W[i, j] for this warp's columns nt*8 + fg, all k-steps
  uint32_t bA[G::NKS][2], bX[G::NKS][2];
  {
    const unsigned short *wa =
        reinterpret_cast<const unsigned short *>(p.W_a) + (size_t)h * kBW * kBW + nt * 8 + fg;
    const unsigned short *wx =
        reinterpret_cast<const unsigned short *>(p.W_x) + (size_t)h * kBW * kBW + nt * 8 + fg;
#pragma unroll
    for (int ks = 0; ks < G::NKS; ++ks)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int kk = ks * 16 + 2 * fq + 8 * hf;
        bA[ks][hf] = pack_bf16(__ldg(wa + (size_t)kk * kBW), __ldg(wa + (size_t)(kk + 1) * kBW));
        bX[ks][hf] = pack_bf16(__ldg(wx + (size_t)kk * kBW), __ldg(wx + (size_t)(kk + 1) * kBW));
      }
  }
  // ldmatrix.x4 row address of this lane: row (l % 8) + 8 ((l / 8) % 2), column 8 (l / 16)
  const uint32_t a_lane = shared_addr(u_s) +
                          (((lane & 7) + ((lane >> 3) & 1) * 8) * G::kStride + (lane >> 4) * 8) * 2;
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (th.active) c = chan_c<T>(p, th.d);
  const float neg_c_sp = -kDecayC * c.sp;
  const int ngt = ceil_div(p.T, kTB);
  const size_t orow = (size_t)b * p.T * D + th.d;
  const float *za_row = z_s + ((th.sl * 2 + 0) * kBW + th.j) * kRow;
  const float *zx_row = z_s + ((th.sl * 2 + 1) * kBW + th.j) * kRow;
  T *u_col = u_s + th.sl * kTB * G::kStride + th.j;
  float P = 1.f, Hl = 0.f, R = 0.f;
  // Staging of group g into ring slot buf: 16-byte copies (kBW / 8 per row) spread
  // over the block. x rows before t = 0 come from the conv history (zeros without
  // one), rows past a segment's end are zero-filled, and segments with no live
  // token in the group are skipped. Every thread commits one group per call
  // (possibly empty), so that cp_async_wait_one_pending always refers to the same
  // group on every thread.
  constexpr int CX = kBW / 8;
  // the dy rows come to exactly one chunk per thread; x rows in a loop of their own,
  // so that a warp's copies stay on one branch
  static_assert(G::S * kTB * CX == G::kThreads, "dy chunks per thread");
  auto stage = [&](int g, int buf) {
    {                                                 // dy row t = tb + k
      const int rowid = threadIdx.x / CX, w = threadIdx.x - rowid * CX;
      const int sl = rowid / kTB, k = rowid - sl * kTB;
      const int s0 = min(p.T, (blockIdx.x * G::S + sl) * pl.L), s1 = min(p.T, s0 + pl.L);
      const int tb = s0 + g * kTB, t = tb + k;
      if (tb < s1)
        cp_async16(dys_st + ((buf * G::S + sl) * kTB + k) * kBW + w * 8,
                   dyb + ((size_t)b * p.T + (t < s1 ? t : tb)) * D + (size_t)h * kBW + w * 8,
                   t < s1);
    }
    for (int ci = threadIdx.x; ci < G::S * XR * CX; ci += G::kThreads) {
      const int rowid = ci / CX, w = ci - rowid * CX;
      const int sl = rowid / XR, r = rowid - sl * XR;
      const int s0 = min(p.T, (blockIdx.x * G::S + sl) * pl.L), s1 = min(p.T, s0 + pl.L);
      const int tb = s0 + g * kTB;
      if (tb >= s1) continue;
      const int t = tb - 3 + r;                       // x row t = tb - 3 + r
      const T *src = xb + (size_t)tb * D + (size_t)h * kBW + w * 8;   // a valid address
      bool full = false;
      if (t >= 0 && t < s1) {
        src = xb + (size_t)t * D + (size_t)h * kBW + w * 8;
        full = true;
      } else if (t < 0 && cs_in_b != nullptr) {
        src = cs_in_b + (size_t)(3 + t) * D + (size_t)h * kBW + w * 8;
        full = true;
      }
      cp_async16(xs_st + ((buf * G::S + sl) * XR + r) * kBW + w * 8, src, full);
    }
    cp_async_commit();
  };
  const int ng = pl.L / kTB;
  stage(0, 0);
  stage(1, 1);
  cp_async_wait_one_pending();
  __syncthreads();
  for (int g = 0; g < ng; ++g) {
    const int tb = th.t0 + g * kTB;
    const bool live = th.active && tb < th.t1;
    const int buf = g % 3;
    float u[kTB];
    if (live) {
      const size_t go = ((size_t)b * ngt + tb / kTB) * D + th.d;
      ws_gP[go] = P;
      ws_gH[go] = Hl;
      // Conv1D from the staged rows (the operation order of conv_group):
      // u_t = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t, rows k .. k + 3
      const T *xr = xs_st + (buf * G::S + th.sl) * XR * kBW + th.j;
      float xw[XR];
#pragma unroll
      for (int r = 0; r < XR; ++r) xw[r] = to_f32<T>(xr[r * kBW]);
#pragma unroll
      for (int k = 0; k < kTB; ++k)
        u[k] = tb + k < th.t1
                   ? fmaf(c.w3, xw[k + 3], fmaf(c.w2, xw[k + 2], fmaf(c.w1, xw[k + 1], c.w0 * xw[k])))
                   : 0.f;
    } else {
#pragma unroll
      for (int k = 0; k < kTB; ++k) u[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < kTB; ++k) u_col[k * G::kStride] = __float2bfloat16_rn(u[k]);
    __syncthreads();
    // ring slot (g + 2) % 3 = (g - 1) % 3 was last read in group g - 1 (its dy rows
    // after that group's second barrier): every thread has passed the barrier above
    stage(g + 2, (g + 2) % 3);
    float acc[2][2][4];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mi][0][e] = acc[mi][1][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < G::NKS; ++ks)
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        uint32_t a[4];
        ldsm_x4(a_lane + ((mt0 + mi) * 16 * G::kStride + ks * 16) * 2, a);
        mma_bf16(acc[mi][0], a, bA[ks][0], bA[ks][1]);
        mma_bf16(acc[mi][1], a, bX[ks][0], bX[ks][1]);
      }
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = (mt0 + mi) * 16 + fg + (e >= 2 ? 8 : 0);
        const int col = nt * 8 + 2 * fq + (e & 1);
        z_s[(((r >> 3) * 2 + 0) * kBW + col) * kRow + (r & 7)] = acc[mi][0][e];
        z_s[(((r >> 3) * 2 + 1) * kBW + col) * kRow + (r & 7)] = acc[mi][1][e];
      }
    cp_async_wait_one_pending();   // group g + 1's rows: published by the barrier below
    __syncthreads();
    if (live) {
      float za[kTB], zx[kTB];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float4 va = reinterpret_cast<const float4 *>(za_row)[q];
        const float4 vx = reinterpret_cast<const float4 *>(zx_row)[q];
        za[4 * q] = va.x + c.ba;
        za[4 * q + 1] = va.y + c.ba;
        za[4 * q + 2] = va.z + c.ba;
        za[4 * q + 3] = va.w + c.ba;
        zx[4 * q] = vx.x + c.bx;
        zx[4 * q + 1] = vx.y + c.bx;
        zx[4 * q + 2] = vx.z + c.bx;
        zx[4 * q + 3] = vx.w + c.bx;
      }
      gates_scan_group<T>(za, zx, u, tb, th.t1, neg_c_sp, dyb, orow, D, P, Hl, R, ws_ga, ws_gx,
                          dys_st + (buf * G::S + th.sl) * kTB * kBW + th.j, kBW);
    }
  }
  cp_async_wait_all();   // no copy outlives the block
  if (!th.active) return;
  const size_t o = ((size_t)b * pl.nseg + th.s) * D + th.d;
  ws_A[o] = P;
  ws_H[o] = Hl;
  ws_R[o] = R;
}

// K2: the two carries as two-level scans of affine maps. A block covers
// kCarryCh channels (one per lane) and splits each channel's segments into
// kCarryParts contiguous parts (one warp per part). Each part composes its
// segments' maps (h -> A h + H forward, c -> A c + R backward) with loads that
// do not depend on one another, the parts' entry values come from folding the
// earlier parts' maps (shared memory), and each part then walks its own
// segments storing h_in and C. The same recurrences as one sequential walk,
// reassociated: the chains are nseg / kCarryParts long instead of nseg.
constexpr int kCarryCh = 32, kCarryParts = 8;
__global__ void __launch_bounds__(kCarryCh * kCarryParts)
bwd_carry_kernel(int B, int D, int nseg, const float *__restrict__ ws_A,
                 const float *__restrict__ ws_H, const float *__restrict__ ws_R,
                 const float *__restrict__ h0, const float *__restrict__ dh_T,
                 float *__restrict__ ws_hin, float *__restrict__ ws_C, float *__restrict__ dh0) {
  __shared__ float mA[kCarryParts][kCarryCh], mV[kCarryParts][kCarryCh];
  const int cl = threadIdx.x % kCarryCh, part = threadIdx.x / kCarryCh;
  const int idx = blockIdx.x * kCarryCh + cl;
  const bool on = idx < B * D;                 // no early return: the block meets at barriers
  const int b = on ? idx / D : 0, d = on ? idx - b * D : 0;
  const int q = ceil_div(nseg, kCarryParts);
  const int s0 = min(nseg, part * q), s1 = min(nseg, s0 + q);
  const size_t base = (size_t)b * nseg * D + d;
  // forward: this part's map h -> Ap h + Vp, then the state entering it
  float Ap = 1.f, Vp = 0.f;
  if (on)
    for (int s = s0; s < s1; ++s) {
      const size_t o = base + (size_t)s * D;
      const float a = ws_A[o];
      Vp = fmaf(a, Vp, ws_H[o]);
      Ap *= a;
    }
  mA[part][cl] = Ap;
  mV[part][cl] = Vp;
  __syncthreads();
  float hh = (on && h0) ? h0[idx] : 0.f;
  for (int r = 0; r < part; ++r) hh = fmaf(mA[r][cl], hh, mV[r][cl]);
  if (on)
    for (int s = s0; s < s1; ++s) {
      const size_t o = base + (size_t)s * D;
      ws_hin[o] = hh;
      hh = fmaf(ws_A[o], hh, ws_H[o]);
    }
  __syncthreads();                             // every part has read mA, mV
  // backward: this part's map c -> Ap c + Vp over its segments last to first,
  // then the gradient entering it from the right
  Ap = 1.f;
  Vp = 0.f;
  if (on)
    for (int s = s1 - 1; s >= s0; --s) {
      const size_t o = base + (size_t)s * D;
      const float a = ws_A[o];
      Vp = fmaf(a, Vp, ws_R[o]);
      Ap *= a;
    }
  mA[part][cl] = Ap;
  mV[part][cl] = Vp;
  __syncthreads();
  float cc = (on && dh_T) ? dh_T[idx] : 0.f;
  for (int r = kCarryParts - 1; r > part; --r) cc = fmaf(mA[r][cl], cc, mV[r][cl]);
  if (on)
    for (int s = s1 - 1; s >= s0; --s) {
      const size_t o = base + (size_t)s * D;
      ws_C[o] = cc;
      cc = fmaf(ws_A[o], cc, ws_R[o]);
    }
  if (on && part == 0 && dh0) dh0[idx] = cc;
}

// The per-thread part of a K3 group (a live thread only): the group's start
// state from (prod a, local state) and h_in, the stored gates r and i, then the reverse
// chain over its tokens. With G_t the state gradient at token t, every
// gradient of the token is G_t times a factor known in time order:
//   d z_a = G c sp (1 - r) Q,  d Lambda-sum term = G c Q,
//   Q = a (a i u (r / g) - h_{t-1} r),
//   d z_x = G g u i (1 - i),   own part of d u = G g i,
// so the forward part keeps five factors per token and the reverse part is a
// handful of multiplies. It writes u, d z_a, d z_x over the workspace, passes
// each token's (d z_a, d z_x) to sink(k, ...) (zeros past t1), leaves the own
// part of d u in dub and advances gc and the per-channel sums (acc_q sums
// G Q; the caller scales it by c).
// kStaged: the group's r, i and dy rows were copied to shared memory ahead
// of time (sr, si, sdy: this thread's channel at token 0 of the group, rows
// sstride elements apart, zeros past t1); else they are read from the
// workspace and dy in global memory, with an L1 prefetch of the next group.
// d W tiles: 64 x 64 (i, j) per block (both d W kernels)
constexpr int kDwTile = 64;

// bf16 copies of u, d z_a and d z_x for the tensor-core d W (which reads its
// operands as bf16): stored by K3 with the same round-to-nearest, so d W is the
// same while these streams move half the bytes of fp32 ones.
struct Bf16Streams {
  __nv_bfloat16 *u, *dza, *dzx;
};

template <typename T, bool kStaged, bool kB16, typename Sink>
__device__ __forceinline__ void final_group(const BwdThread &th, const ChanC &c, const T *xb,
                                            const T *cs_in_b, const T *dyb, size_t orow, int D,
                                            int tb, size_t go, float h_in,
                                            const float *__restrict__ ws_gP,
                                            const float *__restrict__ ws_gH,
                                            float *__restrict__ ws_ga, float *__restrict__ ws_gx,
                                            float *__restrict__ ws_u, float &gc, float &acc_q,
                                            float &acc_ba, float &acc_bx, float (&dub)[kTB],
                                            const float *sr, const float *si, const T *sdy,
                                            const T *sx, const float *sg, int sstride,
                                            const Bf16Streams &b16, Sink sink) {
  const float neg_c_sp = -kDecayC * c.sp, csp = kDecayC * c.sp;
  if (!kStaged && tb - kTB >= th.t0) {
    // the group processed next (8 tokens earlier): its r, i and dy rows
    const float *pga = ws_ga + orow + (size_t)(tb - kTB) * D;
    const float *pgx = ws_gx + orow + (size_t)(tb - kTB) * D;
    const T *pdy = dyb + orow + (size_t)(tb - kTB) * D;
#pragma unroll
    for (int k = 0; k < kTB; ++k) {
      prefetch_l1(pga + (size_t)k * D);
      prefetch_l1(pgx + (size_t)k * D);
      prefetch_l1(pdy + (size_t)k * D);
    }
  }
  float u[kTB], hh;
  if constexpr (kStaged) {
    // the staged x rows tb - 3 .. tb + 7 (conv_group's operation order) and the
    // group's start pair (prod a, local state)
    float xw[kTB + 3];
#pragma unroll
    for (int r = 0; r < kTB + 3; ++r) xw[r] = to_f32<T>(sx[r * sstride]);
#pragma unroll
    for (int k = 0; k < kTB; ++k)
      u[k] = tb + k < th.t1
                 ? fmaf(c.w3, xw[k + 3], fmaf(c.w2, xw[k + 2], fmaf(c.w1, xw[k + 1], c.w0 * xw[k])))
                 : 0.f;
    hh = fmaf(sg[0], h_in, sg[sstride]);
  } else {
    conv_group<T>(xb, cs_in_b, D, th.d, tb, th.t1, c, u);
    hh = fmaf(ws_gP[go], h_in, ws_gH[go]);
  }
  float fa[kTB], fza[kTB], fq[kTB], fzx[kTB], fu[kTB];
#pragma unroll
  for (int k = 0; k < kTB; ++k) {
    const int t = tb + k;
    const size_t o = orow + (size_t)t * D;
    const bool in = t < th.t1;
    float rv, iv;                                 // the gates r and i stored by K1
    if constexpr (kStaged) {
      rv = sr[k * sstride];
      iv = si[k * sstride];
    } else {
      rv = in ? ws_ga[o] : 0.f;
      iv = in ? ws_gx[o] : 0.f;
    }
    if (in) {
      if constexpr (kB16)
        b16.u[o] = __float2bfloat16_rn(u[k]);
      else
        ws_u[o] = u[k];
    }
    const TokGates tg = tok_gates_ri(rv, iv, neg_c_sp);
    const float r = tg.r, ig = tg.i, a = tg.a, gg = tg.g, rog = tg.rog;
    const float q = a * (a * ig * u[k] * rog - hh * r);
    fa[k] = a;
    fq[k] = q;
    fza[k] = csp * (1.f - r) * q;
    fzx[k] = gg * u[k] * ig * (1.f - ig);
    fu[k] = gg * ig;
    hh = fmaf(a, hh, gg * ig * u[k]);
  }
#pragma unroll
  for (int k = kTB - 1; k >= 0; --k) {
    const int t = tb + k;
    float dza = 0.f, dzx = 0.f;
    dub[k] = 0.f;
    if (t < th.t1) {
      const size_t o = orow + (size_t)t * D;
      float dy;
      if constexpr (kStaged) dy = to_f32<T>(sdy[k * sstride]);
      else dy = ldg_f32(dyb + o);
      const float G = dy + gc;
      dza = G * fza[k];
      dzx = G * fzx[k];
      dub[k] = G * fu[k];
      acc_q = fmaf(G, fq[k], acc_q);
      acc_ba += dza;
      acc_bx += dzx;
      gc = fa[k] * G;
      if constexpr (kB16) {
        b16.dza[o] = __float2bfloat16_rn(dza);
        b16.dzx[o] = __float2bfloat16_rn(dzx);
      } else {
        ws_ga[o] = dza;
        ws_gx[o] = dzx;
      }
    }
    sink(k, dza, dzx);
  }
}

template <typename T, bool kSW, int kMaxT>
__global__ void __launch_bounds__(kMaxT, kMaxT == 256 ? 3 : 1)
bwd_final_kernel(BwdArgs p, BwdPlan pl, const float *__restrict__ ws_hin,
                 const float *__restrict__ ws_C, const float *__restrict__ ws_gP,
                 const float *__restrict__ ws_gH, float *__restrict__ ws_ga,
                 float *__restrict__ ws_gx, float *__restrict__ ws_u,
                 float *__restrict__ ws_du) {
  extern __shared__ float4 smem_f[];
  const int bw = p.D / p.H, D = p.D, h = blockIdx.y, b = blockIdx.z;
  float *dz_s = reinterpret_cast<float *>(smem_f);   // [S][2][bw][kRow]: d z_a, d z_x rows
  float *Wsa = dz_s + 2 * pl.S * bw * kRow;          // [bw][bw + 1] when kSW
  float *Wsx = Wsa + (kSW ? bw * (bw + 1) : 0);
  const BwdThread th = bwd_thread(p, pl, bw);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy);
  const T *Wa = static_cast<const T *>(p.W_a) + (size_t)h * bw * bw;
  const T *Wx = static_cast<const T *>(p.W_x) + (size_t)h * bw * bw;
  if (kSW) stage_weights<T>(Wa, Wx, Wsa, Wsx, bw);
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float h_in = 0.f, gc = 0.f;   // gc: a_{t+1} G_{t+1} for the token being processed
  if (th.active) {
    c = chan_c<T>(p, th.d);
    const size_t seg = ((size_t)b * pl.nseg + th.s) * D + th.d;
    h_in = ws_hin[seg];
    gc = ws_C[seg];
  }
  const int ngt = ceil_div(p.T, kTB);
  const int jr = th.j < bw ? th.j : 0;
  const size_t orow = (size_t)b * p.T * D + th.d;
  float *dza_row = dz_s + ((th.sl * 2 + 0) * bw + jr) * kRow;
  float *dzx_row = dz_s + ((th.sl * 2 + 1) * bw + jr) * kRow;
  const float *dza_seg = dz_s + (th.sl * 2 + 0) * bw * kRow;
  const float *dzx_seg = dz_s + (th.sl * 2 + 1) * bw * kRow;
  float acc_q = 0.f, acc_ba = 0.f, acc_bx = 0.f;
  for (int g = pl.L / kTB - 1; g >= 0; --g) {
    const int tb = th.t0 + g * kTB;
    const bool live = th.active && tb < th.t1;
    float dub[kTB];
    if (live) {
      const size_t go = ((size_t)b * ngt + tb / kTB) * D + th.d;
      final_group<T, false, false>(th, c, xb, cs_in_b, dyb, orow, D, tb, go, h_in, ws_gP, ws_gH,
                                   ws_ga, ws_gx, ws_u, gc, acc_q, acc_ba, acc_bx, dub, nullptr,
                                   nullptr, nullptr, nullptr, nullptr, 0, Bf16Streams{},
                                   [&](int k, float dza, float dzx) {
                              dza_row[k] = dza;
                              dzx_row[k] = dzx;
                            });
    } else {
#pragma unroll
      for (int k = 0; k < kTB; ++k) dub[k] = 0.f;
      if (th.j < bw) {
        store_row(dza_row, dub);   // zeros
        store_row(dzx_row, dub);
      }
    }
    __syncthreads();
    if (live) {
      // d u_j += sum_m d z_a[m] W_a[j, m] + d z_x[m] W_x[j, m]
#pragma unroll 8
      for (int m = 0; m < bw; ++m) {
        const float4 a0 = reinterpret_cast<const float4 *>(dza_seg + m * kRow)[0];
        const float4 a1 = reinterpret_cast<const float4 *>(dza_seg + m * kRow)[1];
        const float4 x0 = reinterpret_cast<const float4 *>(dzx_seg + m * kRow)[0];
        const float4 x1 = reinterpret_cast<const float4 *>(dzx_seg + m * kRow)[1];
        const float wa = w_at<T, kSW>(Wa, Wsa, bw, th.j, m);
        const float wx = w_at<T, kSW>(Wx, Wsx, bw, th.j, m);
        const float av[kTB] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float xv[kTB] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int k = 0; k < kTB; ++k) dub[k] = fmaf(av[k], wa, fmaf(xv[k], wx, dub[k]));
      }
#pragma unroll
      for (int k = 0; k < kTB; ++k)
        if (tb + k < th.t1) ws_du[orow + (size_t)(tb + k) * D] = dub[k];
    }
    __syncthreads();
  }
  if (!th.active) return;
  atomicAdd(p.dLambda + th.d, kDecayC * acc_q * (-sigmoid_f32(-__ldg(p.Lambda + th.d))));
  atomicAdd(p.db_a + th.d, acc_ba);
  atomicAdd(p.db_x + th.d, acc_bx);
}

// K3 for bf16 I/O and kBW in {32, 64, 128}: the transposed contraction
// d u += d z_a W_a^T + d z_x W_x^T of each group on the tensor cores. The
// threads put their d z as bf16 rows (token-major) in shared memory, each warp
// multiplies its two m-tiles by its 8 columns of W_a^T and W_x^T into one
// accumulator, scatters it into (segment, channel) rows, and each thread adds
// its channel's 8 tokens to its own part of d u.
template <int kBW>
__global__ void __launch_bounds__(TcGeo<kBW>::kThreads, kBW == 128 ? 1 : 2)
bwd_final_tc_kernel(BwdArgs p, BwdPlan pl, Bf16Streams b16, const float *__restrict__ ws_hin,
                    const float *__restrict__ ws_C, const float *__restrict__ ws_gP,
                    const float *__restrict__ ws_gH, float *__restrict__ ws_ga,
                    float *__restrict__ ws_gx, float *__restrict__ ws_u,
                    float *__restrict__ ws_du) {
  using T = __nv_bfloat16;
  using G = TcGeo<kBW>;
  extern __shared__ float4 smem_ft[];
  float *du_s = reinterpret_cast<float *>(smem_ft);                  // [S][kBW][kRow]
  T *a_s = reinterpret_cast<T *>(du_s + G::S * kBW * kRow);          // [2][M][kStride]
  T *w_s = a_s + 2 * G::M * G::kStride;                              // [2][kBW][kStride]
  // r, i and dy rows of a group, double-buffered: [2][S][kTB][kBW]; then its
  // x rows tb-3 .. tb+7 [2][S][kTB + 3][kBW] and its start pair (prod a, local
  // state) [2][S][2][kBW]
  constexpr int XR = kTB + 3;
  float *ra_st = reinterpret_cast<float *>(w_s + 2 * kBW * G::kStride);
  float *ix_st = ra_st + 2 * G::S * kTB * kBW;
  T *dy_st = reinterpret_cast<T *>(ix_st + 2 * G::S * kTB * kBW);
  T *xs_st = dy_st + 2 * G::S * kTB * kBW;
  float *gs_st = reinterpret_cast<float *>(xs_st + 2 * G::S * XR * kBW);
  const int D = p.D, h = blockIdx.y, b = blockIdx.z;
  const BwdThread th = bwd_thread(p, pl, kBW);
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D;
  const T *cs_in_b =
      p.conv_state_in ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D : nullptr;
  const T *dyb = static_cast<const T *>(p.dy);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nt = (2 * warp) / G::MT, mt0 = (2 * warp) % G::MT;
  const int fg = lane >> 2, fq = lane & 3;
  // The head's W_a and W_x as bf16 rows j (m contiguous, stride kStride) in
  // shared memory: B[k = m][n = j] = W[j, m], so the k pairs of column
  // j = nt*8 + fg are adjacent in row j; read per k-step (2 words per gate).
  {
    const uint32_t *wa = reinterpret_cast<const uint32_t *>(static_cast<const T *>(p.W_a) +
                                                            (size_t)h * kBW * kBW);
    const uint32_t *wx = reinterpret_cast<const uint32_t *>(static_cast<const T *>(p.W_x) +
                                                            (size_t)h * kBW * kBW);
    uint32_t *ws32 = reinterpret_cast<uint32_t *>(w_s);
    for (int idx = threadIdx.x; idx < kBW * kBW / 2; idx += G::kThreads) {
      const int row = idx / (kBW / 2), cw = idx - row * (kBW / 2);
      ws32[row * (G::kStride / 2) + cw] = __ldg(wa + idx);
      ws32[(kBW + row) * (G::kStride / 2) + cw] = __ldg(wx + idx);
    }
  }
  const uint32_t *wfa =
      reinterpret_cast<const uint32_t *>(w_s) + (nt * 8 + fg) * (G::kStride / 2) + fq;
  const uint32_t *wfx = wfa + kBW * (G::kStride / 2);
  const uint32_t a_lane = shared_addr(a_s) +
                          (((lane & 7) + ((lane >> 3) & 1) * 8) * G::kStride + (lane >> 4) * 8) * 2;
  constexpr uint32_t kGateBytes = G::M * G::kStride * 2;   // d z_x rows follow d z_a rows
  ChanC c{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float h_in = 0.f, gc = 0.f;   // gc: a_{t+1} G_{t+1} for the token being processed
  if (th.active) {
    c = chan_c<T>(p, th.d);
    const size_t seg = ((size_t)b * pl.nseg + th.s) * D + th.d;
    h_in = ws_hin[seg];
    gc = ws_C[seg];
  }
  const int ngt = ceil_div(p.T, kTB);
  const size_t orow = (size_t)b * p.T * D + th.d;
  T *dza_col = a_s + th.sl * kTB * G::kStride + th.j;
  T *dzx_col = dza_col + G::M * G::kStride;
  const float *du_row = du_s + (th.sl * kBW + th.j) * kRow;
  float acc_q = 0.f, acc_ba = 0.f, acc_bx = 0.f;
  // Staging of group g's rows into buffer buf: 16-byte copies spread over the
  // block (per segment and token: kBW/4 chunks of z_a, kBW/4 of z_x, kBW/8 of
  // dy; per segment: 11 x rows of kBW/8 chunks and 2 start-pair rows of kBW/4).
  // Rows past a segment's end are zero-filled, x rows before t = 0 come from the
  // conv history (zeros without one); segments with no live token in the group
  // are skipped (no thread reads them).
  constexpr int CZ = kBW / 4, CY = kBW / 8, CXG = XR * CY + 2 * CZ;
  // z_a and z_x rows come to exactly two chunks per thread each, dy rows to one;
  // one loop per stream keeps a warp's copies on one branch
  static_assert(G::S * kTB * CZ == 2 * G::kThreads && G::S * kTB * CY == G::kThreads,
                "chunks per thread");
  auto stage = [&](int g, int buf) {
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int ci = threadIdx.x + (q < 2 ? q : 0) * G::kThreads;
      const int cpr = q < 2 ? CZ : CY;                // chunks per row (powers of two)
      const int rowid = ci / cpr, w = ci - rowid * cpr;
      const int sl = rowid / kTB, k = rowid - sl * kTB;
      const int s0 = min(p.T, (blockIdx.x * G::S + sl) * pl.L), s1 = min(p.T, s0 + pl.L);
      const int tb = s0 + g * kTB;
      if (tb >= s1) continue;
      const bool in = tb + k < s1;
      const size_t grow = ((size_t)b * p.T + (in ? tb + k : tb)) * D + (size_t)h * kBW;
      const int slot = ((buf * G::S + sl) * kTB + k) * kBW;
      if (q < 2) {
        cp_async16(ra_st + slot + w * 4, ws_ga + grow + w * 4, in);
        cp_async16(ix_st + slot + w * 4, ws_gx + grow + w * 4, in);
        continue;
      }
      cp_async16(dy_st + slot + w * 8, dyb + grow + w * 8, in);
    }
    for (int ci = threadIdx.x; ci < G::S * CXG; ci += G::kThreads) {
      const int sl = ci / CXG, w = ci - sl * CXG;
      const int s0 = min(p.T, (blockIdx.x * G::S + sl) * pl.L), s1 = min(p.T, s0 + pl.L);
      const int tb = s0 + g * kTB;
      if (tb >= s1) continue;
      if (w < XR * CY) {                              // x row t = tb - 3 + r
        const int r = w / CY, cx = w - r * CY, t = tb - 3 + r;
        const size_t col = (size_t)h * kBW + cx * 8;
        const T *src = xb + (size_t)tb * D + col;     // a valid address
        bool full = false;
        if (t >= 0 && t < s1) {
          src = xb + (size_t)t * D + col;
          full = true;
        } else if (t < 0 && cs_in_b != nullptr) {
          src = cs_in_b + (size_t)(3 + t) * D + col;
          full = true;
        }
        cp_async16(xs_st + ((buf * G::S + sl) * XR + r) * kBW + cx * 8, src, full);
      } else {                                        // prod a (row 0), local state (row 1)
        const int w2 = w - XR * CY, which = w2 / CZ, cz = w2 - which * CZ;
        const size_t go = ((size_t)b * ngt + tb / kTB) * D + (size_t)h * kBW + cz * 4;
        cp_async16(gs_st + ((buf * G::S + sl) * 2 + which) * kBW + cz * 4,
                   (which ? ws_gH : ws_gP) + go, true);
      }
    }
    cp_async_commit();
  };
  const int ng = pl.L / kTB;
  stage(ng - 1, 0);
  cp_async_wait_all();
  __syncthreads();
  for (int g = ng - 1; g >= 0; --g) {
    const int tb = th.t0 + g * kTB;
    const bool live = th.active && tb < th.t1;
    const int buf = (ng - 1 - g) & 1;
    // the next group's rows land while this group is computed (its buffer was
    // last read before the previous iteration's barriers)
    if (g > 0) stage(g - 1, buf ^ 1);
    float dub[kTB];
    if (live) {
      const size_t go = ((size_t)b * ngt + tb / kTB) * D + th.d;
      const int srow = ((buf * G::S + th.sl) * kTB) * kBW + th.j;
      final_group<T, true, kBW % kDwTile == 0>(th, c, xb, cs_in_b, dyb, orow, D, tb, go, h_in,
                                               ws_gP, ws_gH, ws_ga, ws_gx, ws_u, gc, acc_q,
                                               acc_ba, acc_bx, dub, ra_st + srow, ix_st + srow,
                                               dy_st + srow,
                                               xs_st + (buf * G::S + th.sl) * XR * kBW + th.j,
                                               gs_st + (buf * G::S + th.sl) * 2 * kBW + th.j,
                                               kBW, b16,
                                               [&](int k, float dza, float dzx) {
                             dza_col[k * G::kStride] = __float2bfloat16_rn(dza);
                             dzx_col[k * G::kStride] = __float2bfloat16_rn(dzx);
                           });
    } else {
#pragma unroll
      for (int k = 0; k < kTB; ++k) {
        dub[k] = 0.f;
        dza_col[k * G::kStride] = __float2bfloat16_rn(0.f);
        dzx_col[k * G::kStride] = __float2bfloat16_rn(0.f);
      }
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mi][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < G::NKS; ++ks) {
      // elements ks*16 + 2 fq + 8 hf of row j: words ks*8 + fq + 4 hf
      const uint32_t ba0 = wfa[ks * 8], ba1 = wfa[ks * 8 + 4];
      const uint32_t bx0 = wfx[ks * 8], bx1 = wfx[ks * 8 + 4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const uint32_t off = ((mt0 + mi) * 16 * G::kStride + ks * 16) * 2;
        uint32_t a[4];
        ldsm_x4(a_lane + off, a);
        mma_bf16(acc[mi], a, ba0, ba1);
        ldsm_x4(a_lane + kGateBytes + off, a);
        mma_bf16(acc[mi], a, bx0, bx1);
      }
    }
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = (mt0 + mi) * 16 + fg + (e >= 2 ? 8 : 0);
        const int col = nt * 8 + 2 * fq + (e & 1);
        du_s[((r >> 3) * kBW + col) * kRow + (r & 7)] = acc[mi][e];
      }
    cp_async_wait_all();   // the next group's rows: published by the barrier below
    __syncthreads();
    if (live) {
      const float4 v0 = reinterpret_cast<const float4 *>(du_row)[0];
      const float4 v1 = reinterpret_cast<const float4 *>(du_row)[1];
      const float dv[kTB] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int k = 0; k < kTB; ++k)
        if (tb + k < th.t1) ws_du[orow + (size_t)(tb + k) * D] = dub[k] + dv[k];
    }
  }
  if (!th.active) return;
  atomicAdd(p.dLambda + th.d, kDecayC * acc_q * (-sigmoid_f32(-__ldg(p.Lambda + th.d))));
  atomicAdd(p.db_a + th.d, acc_ba);
  atomicAdd(p.db_x + th.d, acc_bx);
}

// d W[h, i, j] += sum_n U[n, h bw + i] dZ[n, h bw + j] over one chunk of
// tokens: a 64 x 64 tile of (i, j) of one gate and head per block, 4 x 4 per
// thread, 32 tokens of both operands staged in shared memory at a time (the
// next 32 already in flight to registers).
constexpr int kDwRows = 32, kDwThreads = 256;

__global__ void __launch_bounds__(kDwThreads)
bwd_dw_kernel(const float *__restrict__ U, const float *__restrict__ dZa,
              const float *__restrict__ dZx, float *__restrict__ dWa, float *__restrict__ dWx,
              int N, int D, int H, int chunk) {
  __shared__ __align__(16) float us[kDwRows][kDwTile];
  __shared__ __align__(16) float zs[kDwRows][kDwTile];
  const int bw = D / H;
  const int tiles = ceil_div(bw, kDwTile);
  int tile = blockIdx.x;
  const int gate = tile & 1;
  tile >>= 1;
  const int ti = tile % tiles, tj = (tile / tiles) % tiles, h = tile / (tiles * tiles);
  const float *Z = gate == 0 ? dZa : dZx;
  float *dW = gate == 0 ? dWa : dWx;
  const int tid = threadIdx.x;
  const int ri = tid >> 4, rj = tid & 15;   // this thread's rows 4 ri.., columns 4 rj..
  const int lc = tid & 63, lr = tid >> 6;   // loader: column lc, rows lr + 4 q
  const int i0 = ti * kDwTile, j0 = tj * kDwTile;
  const bool iok = i0 + lc < bw, jok = j0 + lc < bw;
  const float *Uc = U + (size_t)h * bw + i0 + lc;
  const float *Zc = Z + (size_t)h * bw + j0 + lc;
  const int n_begin = blockIdx.y * chunk, n_end = min(N, n_begin + chunk);
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[a][e] = 0.f;
  // the next 32 tokens' loads are issued before this tile's FMAs (register prefetch)
  float pu[kDwRows / 4], pz[kDwRows / 4];
  auto fetch = [&](int n0) {
#pragma unroll
    for (int q = 0; q < kDwRows / 4; ++q) {
      const int n = n0 + lr + 4 * q;
      const bool ok = n < n_end;
      pu[q] = ok && iok ? Uc[(size_t)n * D] : 0.f;
      pz[q] = ok && jok ? Zc[(size_t)n * D] : 0.f;
    }
  };
  fetch(n_begin);
  for (int n0 = n_begin; n0 < n_end; n0 += kDwRows) {
#pragma unroll
    for (int q = 0; q < kDwRows / 4; ++q) {
      us[lr + 4 * q][lc] = pu[q];
      zs[lr + 4 * q][lc] = pz[q];
    }
    __syncthreads();
    if (n0 + kDwRows < n_end) fetch(n0 + kDwRows);
#pragma unroll 4
    for (int nn = 0; nn < kDwRows; ++nn) {
      const float4 uv = *reinterpret_cast<const float4 *>(&us[nn][4 * ri]);
      const float4 zv = *reinterpret_cast<const float4 *>(&zs[nn][4 * rj]);
      const float ua[4] = {uv.x, uv.y, uv.z, uv.w};
      const float za[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][e] = fmaf(ua[a], za[e], acc[a][e]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + 4 * ri + a, jj = j0 + 4 * rj + e;
      if (i < bw && jj < bw) atomicAdd(dW + ((size_t)h * bw + i) * bw + jj, acc[a][e]);
    }
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}

// d W on the tensor cores (bf16 I/O, heads a multiple of 64 wide): the same
// 64 x 64 (i, j) tiles and token chunks as bwd_dw_kernel, 4 warps each a
// 32 x 32 quarter. kDwTcRows tokens of U and dZ are staged as bf16 token-major rows
// (padded by 8 elements); with A[i][n] = U[n][i] and B[n][j] = dZ[n][j], both
// fragments come from ldmatrix .trans of those rows (a thread receives stored
// elements (2q, g) and (2q + 1, g) of each 8 x 8 block: the k pairs of column
// g). The rows arrive by 16-byte cp.async through a ring of kDwTcStages steps
// (kDwTcStages - 1 steps in flight during the MMAs), with no staging registers.
constexpr int kDwTcThreads = 128, kDwTcStride = kDwTile + 8;
// tokens per step of the tensor-core d W: 64, so that a block's loads of the next step
// cover twice the bytes of the CUDA-core kernel's 32-token steps
constexpr int kDwTcRows = 64, kDwTcStages = 3;

__global__ void __launch_bounds__(kDwTcThreads)
bwd_dw_tc_kernel(const __nv_bfloat16 *__restrict__ U, const __nv_bfloat16 *__restrict__ dZa,
                 const __nv_bfloat16 *__restrict__ dZx, float *__restrict__ dWa,
                 float *__restrict__ dWx, int N, int D, int H, int chunk) {
  extern __shared__ uint4 dw_sm[];
  // [kDwTcStages][kDwTcRows][kDwTcStride] bf16 each
  __nv_bfloat16 *us = reinterpret_cast<__nv_bfloat16 *>(dw_sm);
  __nv_bfloat16 *zs = us + kDwTcStages * kDwTcRows * kDwTcStride;
  const int bw = D / H;
  const int tiles = bw / kDwTile;
  int tile = blockIdx.x;
  const int gate = tile & 1;
  tile >>= 1;
  const int ti = tile % tiles, tj = (tile / tiles) % tiles, h = tile / (tiles * tiles);
  const __nv_bfloat16 *Z = gate == 0 ? dZa : dZx;
  float *dW = gate == 0 ? dWa : dWx;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wi = (warp & 1) * 32, wj = (warp >> 1) * 32;
  const int i0 = ti * kDwTile, j0 = tj * kDwTile;
  const __nv_bfloat16 *Ub = U + (size_t)h * bw + i0;
  const __nv_bfloat16 *Zb = Z + (size_t)h * bw + j0;
  const int n_begin = blockIdx.y * chunk, n_end = min(N, n_begin + chunk);
  // step s (tokens n_begin + s * kDwTcRows ...) into ring stage s % kDwTcStages:
  // 8 chunks of 16 bytes per row and operand, rows past n_end zero-filled; one
  // commit per call, also for steps past the chunk
  constexpr int kChunks = kDwTcRows * 8 / kDwTcThreads;
  static_assert(kDwTcRows * 8 % kDwTcThreads == 0, "chunks per thread");
  auto issue = [&](int step) {
    const int n0 = n_begin + step * kDwTcRows, stg = step % kDwTcStages;
    if (n0 < n_end) {
#pragma unroll
      for (int q = 0; q < kChunks; ++q) {
        const int c = tid + q * kDwTcThreads, r = c >> 3, col = (c & 7) * 8;
        const int n = n0 + r;
        const bool ok = n < n_end;
        const size_t row = (size_t)(ok ? n : n_begin) * D + col;
        const int dst = (stg * kDwTcRows + r) * kDwTcStride + col;
        cp_async16(us + dst, Ub + row, ok);
        cp_async16(zs + dst, Zb + row, ok);
      }
    }
    cp_async_commit();
  };
  // ldmatrix lane rows: A blocks (n-block q / 2, i-block q % 2), B blocks (n-block q % 2,
  // j-block q / 2), q = lane / 8
  const int lq = lane >> 3, lrow = lane & 7;
  const uint32_t a_lane0 =
      shared_addr(us + (lrow + (lq >> 1) * 8) * kDwTcStride + wi + (lq & 1) * 8);
  const uint32_t b_lane0 =
      shared_addr(zs + (lrow + (lq & 1) * 8) * kDwTcStride + wj + (lq >> 1) * 8);
  constexpr uint32_t kRowBytes = kDwTcStride * 2;
  constexpr uint32_t kStageBytes = kDwTcRows * kRowBytes;
  float acc[2][4][4];
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mi][nt][e] = 0.f;
  const int nsteps = n_end > n_begin ? ceil_div(n_end - n_begin, kDwTcRows) : 0;
#pragma unroll
  for (int st = 0; st < kDwTcStages - 1; ++st) issue(st);
  for (int it = 0; it < nsteps; ++it) {
    // stage (it + kDwTcStages - 1) % kDwTcStages was last read in step it - 1, before
    // that step's closing barrier
    issue(it + kDwTcStages - 1);
    asm volatile("cp.async.wait_group %0;" ::"n"(kDwTcStages - 1) : "memory");  // step it
    __syncthreads();
    const uint32_t a_lane = a_lane0 + (it % kDwTcStages) * kStageBytes;
    const uint32_t b_lane = b_lane0 + (it % kDwTcStages) * kStageBytes;
#pragma unroll
    for (int ks = 0; ks < kDwTcRows / 16; ++ks) {
      uint32_t a[2][4], b[2][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) ldsm_x4_trans(a_lane + ks * 16 * kRowBytes + mi * 32, a[mi]);
#pragma unroll
      for (int np = 0; np < 2; ++np) ldsm_x4_trans(b_lane + ks * 16 * kRowBytes + np * 32, b[np]);
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
          mma_bf16(acc[mi][nt], a[mi], b[nt >> 1][(nt & 1) * 2], b[nt >> 1][(nt & 1) * 2 + 1]);
    }
    __syncthreads();
  }
  cp_async_wait_all();   // the empty groups past the chunk
  const int fg = lane >> 2, fq = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + wi + mi * 16 + fg + (e >= 2 ? 8 : 0);
        const int jj = j0 + wj + nt * 8 + 2 * fq + (e & 1);
        atomicAdd(dW + ((size_t)h * bw + i) * bw + jj, acc[mi][nt][e]);
      }
}

// Two adjacent channels of the I/O type as floats (p 2-element aligned), and back.
template <typename T>
__device__ __forceinline__ float2 ldg_pair(const T *p);
template <>
__device__ __forceinline__ float2 ldg_pair<float>(const float *p) {
  return __ldg(reinterpret_cast<const float2 *>(p));
}
template <>
__device__ __forceinline__ float2 ldg_pair<__nv_bfloat16>(const __nv_bfloat16 *p) {
  const unsigned int w = __ldg(reinterpret_cast<const unsigned int *>(p));
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
}
template <typename T>
__device__ __forceinline__ void st_pair(T *p, float2 v);
template <>
__device__ __forceinline__ void st_pair<float>(float *p, float2 v) {
  *reinterpret_cast<float2 *>(p) = v;
}
template <>
__device__ __forceinline__ void st_pair<__nv_bfloat16>(__nv_bfloat16 *p, float2 v) {
  *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v.x, v.y);
}
// A pair as it lies in memory (two bf16 in one word, or two floats) as floats.
template <typename T>
__device__ __forceinline__ float2 pair_to_f2(
    typename std::conditional<sizeof(T) == 2, uint32_t, float2>::type v);
template <>
__device__ __forceinline__ float2 pair_to_f2<float>(float2 v) {
  return v;
}
template <>
__device__ __forceinline__ float2 pair_to_f2<__nv_bfloat16>(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
}

// d x (and the conv history's gradient) from d u, and d w per channel, for one
// chunk of kConvChunk extended positions m (x_{m-3}) of one batch row; thread
// per two adjacent channels, the last three d u values in registers:
//   d x_{m-3} = sum_k w[k] d u_{m-k},  d w[k] += x_{m-3} d u_{m-k}  (0 <= m-k < T).
// Each thread streams its own d u pairs (8 B) and x pairs (4 or 8 B) through a
// private ring of kConvStages batches of kConvBatch positions in shared memory
// (cp.async, kConvStages - 1 batches ahead): many loads in flight per thread at
// no register cost, and no block barrier, as no thread reads another's slots.
constexpr int kConvChunk = 64, kConvThreads = 256, kConvBatch = 8, kConvStages = 2;

// cp.async of n = 4 or 8 bytes (.ca), zero-filled when !full (src must still be
// a valid address); completed by cp.async.wait_group on the issuing thread.
template <int n>
__device__ __forceinline__ void cp_async_small(void *dst, const void *src, bool full) {
  static_assert(n == 4 || n == 8, "cp.async .ca size");
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(shared_addr(dst)),
               "l"(src), "n"(n), "r"(full ? n : 0)
               : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads)
bwd_conv_kernel(BwdArgs p, const float *__restrict__ du) {
  using X2 = typename std::conditional<sizeof(T) == 2, uint32_t, float2>::type;  // an x pair
  extern __shared__ float2 conv_sm[];
  float2 *s_du = conv_sm;                                         // [stage][batch][thread]
  X2 *s_x = reinterpret_cast<X2 *>(s_du + kConvStages * kConvBatch * kConvThreads);
  const int D = p.D;
  const int d = 2 * (blockIdx.x * kConvThreads + threadIdx.x);   // D is a multiple of 8
  const int b = blockIdx.y;
  if (d >= D) return;                 // no barriers below: each thread works on its own
  const int m_begin = blockIdx.z * kConvChunk, m_end = min(p.T + 3, m_begin + kConvChunk);
  const T *cw = static_cast<const T *>(p.conv_w);
  float2 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = ldg_pair<T>(cw + (size_t)k * D + d);
  const float *dub = du + (size_t)b * p.T * D + d;
  const T *xb = static_cast<const T *>(p.x) + (size_t)b * p.T * D + d;
  const T *csb = p.conv_state_in
                     ? static_cast<const T *>(p.conv_state_in) + (size_t)b * 3 * D + d
                     : nullptr;
  T *dxb = static_cast<T *>(p.dx) + (size_t)b * p.T * D + d;
  auto du_at = [&](int t) {
    return (t >= 0 && t < p.T) ? __ldg(reinterpret_cast<const float2 *>(dub + (size_t)t * D))
                               : make_float2(0.f, 0.f);
  };
  // batch j of the chunk into ring stage j % kConvStages: d u_m and x_{m-3} for its
  // positions m (zeros past T, the conv history or zeros before t = 0); one commit
  // per call, also when the batch lies past the chunk
  auto issue = [&](int j) {
    const int stg = j % kConvStages;
#pragma unroll
    for (int i = 0; i < kConvBatch; ++i) {
      const int m = m_begin + j * kConvBatch + i;
      if (m >= m_end) break;
      const int slot = (stg * kConvBatch + i) * kConvThreads + threadIdx.x;
      const bool gin = m < p.T;
      cp_async_small<8>(s_du + slot, gin ? dub + (size_t)m * D : dub, gin);
      const int t = m - 3;
      const T *xs = xb;
      bool xin = false;
      if (t >= 0) {
        xs = xb + (size_t)t * D;
        xin = true;
      } else if (csb != nullptr) {
        xs = csb + (size_t)(3 + t) * D;
        xin = true;
      }
      cp_async_small<sizeof(X2)>(s_x + slot, xs, xin);
    }
    cp_async_commit();
  };
  float2 g1 = du_at(m_begin - 1), g2 = du_at(m_begin - 2), g3 = du_at(m_begin - 3);
  float2 dw[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) dw[k] = make_float2(0.f, 0.f);
  const int nb = ceil_div(m_end - m_begin, kConvBatch);
#pragma unroll
  for (int j = 0; j < kConvStages - 1; ++j) issue(j);
  for (int j = 0; j < nb; ++j) {
    // stage (j + kConvStages - 1) % kConvStages was read by this thread in batch j - 1
    issue(j + kConvStages - 1);
    asm volatile("cp.async.wait_group %0;" ::"n"(kConvStages - 1) : "memory");  // batch j landed
    const int stg = j % kConvStages;
#pragma unroll
    for (int i = 0; i < kConvBatch; ++i) {
      const int m = m_begin + j * kConvBatch + i;
      if (m >= m_end) break;
      const int slot = (stg * kConvBatch + i) * kConvThreads + threadIdx.x;
      const float2 g0 = s_du[slot];
      const float2 xv = pair_to_f2<T>(s_x[slot]);
      float2 acc;
      acc.x = fmaf(w[0].x, g0.x, fmaf(w[1].x, g1.x, fmaf(w[2].x, g2.x, w[3].x * g3.x)));
      acc.y = fmaf(w[0].y, g0.y, fmaf(w[1].y, g1.y, fmaf(w[2].y, g2.y, w[3].y * g3.y)));
      dw[0].x = fmaf(xv.x, g0.x, dw[0].x);
      dw[0].y = fmaf(xv.y, g0.y, dw[0].y);
      dw[1].x = fmaf(xv.x, g1.x, dw[1].x);
      dw[1].y = fmaf(xv.y, g1.y, dw[1].y);
      dw[2].x = fmaf(xv.x, g2.x, dw[2].x);
      dw[2].y = fmaf(xv.y, g2.y, dw[2].y);
      dw[3].x = fmaf(xv.x, g3.x, dw[3].x);
      dw[3].y = fmaf(xv.y, g3.y, dw[3].y);
      if (m >= 3) st_pair<T>(dxb + (size_t)(m - 3) * D, acc);
      else if (p.dconv_state_in)
        *reinterpret_cast<float2 *>(p.dconv_state_in + ((size_t)b * 3 + m) * D + d) = acc;
      g3 = g2;
      g2 = g1;
      g1 = g0;
    }
  }
  cp_async_wait_all();   // the empty groups past the chunk
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    atomicAdd(p.dconv_w + (size_t)k * D + d, dw[k].x);
    atomicAdd(p.dconv_w + (size_t)k * D + d + 1, dw[k].y);
  }
}

struct BwdLayout {
  size_t off_A, off_H, off_R, off_hin, off_C, off_gP, off_gH, off_ga, off_gx, off_u, off_du;
  size_t off_dzx16;   // bf16 d z_x for the tensor-core d W (bf16 u and d z_a share u's region)
  size_t total;
};

BwdLayout bwd_layout(int B, int T, int D, int H) {
  const BwdPlan pl = bwd_plan(B, T, D, H);
  const size_t seg = align_up((size_t)B * pl.nseg * D * sizeof(float), 256);
  const size_t grp = align_up((size_t)B * ceil_div(T, kTB) * D * sizeof(float), 256);
  const size_t tok = align_up((size_t)B * T * D * sizeof(float), 256);
  BwdLayout L{};
  L.off_A = 0;
  L.off_H = L.off_A + seg;
  L.off_R = L.off_H + seg;
  L.off_hin = L.off_R + seg;
  L.off_C = L.off_hin + seg;
  L.off_gP = L.off_C + seg;
  L.off_gH = L.off_gP + grp;
  L.off_ga = L.off_gH + grp;
  L.off_gx = L.off_ga + tok;
  L.off_u = L.off_gx + tok;
  L.off_du = L.off_u + tok;
  L.off_dzx16 = L.off_du + tok;
  L.total = L.off_dzx16 + align_up((size_t)B * T * D * 2, 256);
  return L;
}

// kTcBW > 0: bf16 I/O with heads kTcBW wide, K1 and K3 on the tensor cores.
template <typename T, bool kSW, int kMaxT, int kTcBW>
cudaError_t launch_bwd_t(const BwdArgs &p, void *ws, cudaStream_t st) {
  const int bw = p.D / p.H;
  const BwdPlan pl = bwd_plan(p.B, p.T, p.D, p.H);
  const BwdLayout Ly = bwd_layout(p.B, p.T, p.D, p.H);
  unsigned char *w = static_cast<unsigned char *>(ws);
  auto at = [w](size_t off) { return reinterpret_cast<float *>(w + off); };
  float *A = at(Ly.off_A), *Hh = at(Ly.off_H), *R = at(Ly.off_R);
  float *hin = at(Ly.off_hin), *C = at(Ly.off_C), *gP = at(Ly.off_gP), *gH = at(Ly.off_gH);
  // ga, gx: the gates r and i per token from K1; K3 writes d z_a and d z_x over them
  // for the CUDA-core d W
  float *ga = at(Ly.off_ga), *gx = at(Ly.off_gx), *U = at(Ly.off_u), *du = at(Ly.off_du);
  // bf16 u, d z_a (in u's fp32 region, two halves) and d z_x for the tensor-core d W
  const size_t ntok = (size_t)p.B * p.T * p.D;
  Bf16Streams b16{reinterpret_cast<__nv_bfloat16 *>(U), reinterpret_cast<__nv_bfloat16 *>(U) + ntok,
                  reinterpret_cast<__nv_bfloat16 *>(w + Ly.off_dzx16)};
  const size_t D = p.D;
  cudaError_t e;
  // the accumulated gradients start at zero
  if ((e = cudaMemsetAsync(p.dconv_w, 0, 4 * D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dW_a, 0, D * bw * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dW_x, 0, D * bw * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.db_a, 0, D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.db_x, 0, D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dLambda, 0, D * sizeof(float), st)) != cudaSuccess) return e;

  const int threads = pl.S * pl.bwp;
  const dim3 grid(ceil_div(pl.nseg, pl.S), p.H, p.B);
  const int bd = p.B * p.D;
  if constexpr (kTcBW > 0) {
    using G = TcGeo<kTcBW>;
    // K1: fp32 z rows [S][2][bw][kRow], bf16 u rows [M][kStride] and the staged
    //     x and dy rows (bf16) [3][S][2 kTB + 3][bw];
    // K3: fp32 d u rows [S][bw][kRow], bf16 d z_a, d z_x rows [2][M][kStride],
    //     bf16 W_a, W_x rows [2][bw][kStride], the staged r, i (fp32) and dy
    //     (bf16) rows [2][S][kTB][bw], x rows (bf16) [2][S][kTB + 3][bw] and start
    //     pairs (fp32) [2][S][2][bw]
    const size_t smem1 = (size_t)G::S * 2 * kTcBW * kRow * 4 + (size_t)G::M * G::kStride * 2 +
                         3 * (size_t)G::S * (2 * kTB + 3) * kTcBW * 2;
    const size_t smem3 = (size_t)G::S * kTcBW * kRow * 4 + 2 * (size_t)G::M * G::kStride * 2 +
                         2 * (size_t)kTcBW * G::kStride * 2 +   // + bf16 W_a, W_x rows
                         2 * (size_t)G::S * kTB * kTcBW * (4 + 4 + 2) +   // + staged rows
                         2 * (size_t)G::S * (kTB + 3) * kTcBW * 2 +       // + staged x rows
                         2 * (size_t)G::S * 2 * kTcBW * 4;                // + start pairs
    if ((e = cudaFuncSetAttribute(bwd_gates_tc_kernel<kTcBW>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_final_tc_kernel<kTcBW>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3)) !=
        cudaSuccess)
      return e;
    bwd_gates_tc_kernel<kTcBW><<<grid, G::kThreads, smem1, st>>>(p, pl, A, Hh, R, gP, gH, ga, gx);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_carry_kernel<<<ceil_div(bd, kCarryCh), kCarryCh * kCarryParts, 0, st>>>(
        p.B, p.D, pl.nseg, A, Hh, R, p.h0, p.dh_T, hin, C, p.dh0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_final_tc_kernel<kTcBW><<<grid, G::kThreads, smem3, st>>>(p, pl, b16, hin, C, gP, gH, ga,
                                                                  gx, U, du);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    const size_t wsm = kSW ? 2 * (size_t)bw * (bw + 1) * sizeof(float) : 0;
    // K1: double-buffered u rows; K3: d z_a and d z_x rows; both [S][bw][kRow]
    const size_t smem1 = 2 * (size_t)pl.S * bw * kRow * sizeof(float) + wsm;
    const size_t smem3 = smem1;
    if ((e = cudaFuncSetAttribute(bwd_gates_kernel<T, kSW, kMaxT>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_final_kernel<T, kSW, kMaxT>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3)) !=
        cudaSuccess)
      return e;
    bwd_gates_kernel<T, kSW, kMaxT><<<grid, threads, smem1, st>>>(p, pl, A, Hh, R, gP, gH, ga,
                                                                   gx);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_carry_kernel<<<ceil_div(bd, kCarryCh), kCarryCh * kCarryParts, 0, st>>>(
        p.B, p.D, pl.nseg, A, Hh, R, p.h0, p.dh_T, hin, C, p.dh0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_final_kernel<T, kSW, kMaxT><<<grid, threads, smem3, st>>>(p, pl, hin, C, gP, gH, ga, gx,
                                                                   U, du);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // K4: about 8 blocks of 256 threads per SM of a 148-SM part over the token chunks
  const int N = p.B * p.T;
  const int tiles = ceil_div(bw, kDwTile);
  const int tile_blocks = 2 * tiles * tiles * p.H;
  const bool dw_tc = kTcBW > 0 && kTcBW % kDwTile == 0;
  // token chunks for about 8 blocks per SM, 4 for the tensor-core kernel (its ring
  // of shared memory holds 4 per SM): one wave
  const int nchunk = ceil_div((dw_tc ? 4 : 8) * 148, tile_blocks);
  const int dw_rows = dw_tc ? kDwTcRows : kDwRows;   // tokens per step
  const int chunk = ceil_div(ceil_div(N, nchunk), dw_rows) * dw_rows;
  if (dw_tc) {
    const size_t smem_dw = (size_t)kDwTcStages * 2 * kDwTcRows * kDwTcStride * 2;
    if ((e = cudaFuncSetAttribute(bwd_dw_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_dw)) != cudaSuccess)
      return e;
    bwd_dw_tc_kernel<<<dim3(tile_blocks, ceil_div(N, chunk)), kDwTcThreads, smem_dw, st>>>(
        b16.u, b16.dza, b16.dzx, p.dW_a, p.dW_x, N, p.D, p.H, chunk);
  } else
    bwd_dw_kernel<<<dim3(tile_blocks, ceil_div(N, chunk)), kDwThreads, 0, st>>>(
        U, ga, gx, p.dW_a, p.dW_x, N, p.D, p.H, chunk);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem_conv = (size_t)kConvStages * kConvBatch * kConvThreads * (8 + 2 * sizeof(T));
  if ((e = cudaFuncSetAttribute(bwd_conv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_conv)) != cudaSuccess)
    return e;
  bwd_conv_kernel<T><<<dim3(ceil_div(p.D, 2 * kConvThreads), p.B,
                            ceil_div(p.T + 3, kConvChunk)),
                       kConvThreads, smem_conv, st>>>(p, du);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_io(const BwdArgs &p, void *ws, cudaStream_t st) {
  const int bw = p.D / p.H;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // bf16 operands for the two in-loop gate contractions (tensor cores), from
    // one 8-token group over all rows up: below that a channel has fewer than
    // 8 samples, and the operands' rounding (2^-9 of u and of d z), against
    // cancellation between d u's two terms, is no longer small next to the
    // channel's own scale; those tiny problems take the fp32 operands below
    if (static_cast<long long>(p.B) * p.T >= 8) {
      if (bw == 32) return launch_bwd_t<T, false, 256, 32>(p, ws, st);
      if (bw == 64) return launch_bwd_t<T, false, 256, 64>(p, ws, st);
      if (bw == 128) return launch_bwd_t<T, false, 512, 128>(p, ws, st);
    }
  }
  // both gate weights in shared memory (fp32) up to 128-wide heads: 2 x 129 x 128 x 4 B;
  // a segment's threads (bw rounded up to a warp) fit a 512-thread block up to 512-wide
  // heads; heads up to 64 wide run 256-thread blocks, several per SM
  if (bw <= 64) return launch_bwd_t<T, true, 256, 0>(p, ws, st);
  if (bw <= 128) return launch_bwd_t<T, true, 512, 0>(p, ws, st);
  if (bw <= 512) return launch_bwd_t<T, false, 512, 0>(p, ws, st);
  return launch_bwd_t<T, false, 1024, 0>(p, ws, st);
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int D, int H) { return bwd_layout(B, T, D, H).total; }

int bwd_launches() { return 5; }

cudaError_t launch_bwd(const BwdArgs &p, int io, void *ws, cudaStream_t st) {
  if (io == RGLRU_IO_F32) return launch_bwd_io<float>(p, ws, st);
  return launch_bwd_io<__nv_bfloat16>(p, ws, st);
}

}  // namespace rglru
