// Fused RG-LRU forward on the 5th-generation tensor core (sm_100a), bf16 I/O.
//
// One pass over HBM: x is read once (TMA), y written once. The layer
// ("Griffin: Mixing Gated Linear Recurrences with Local Attention for Efficient
// Language Models", section "Model Architecture"; gates independent of the
// state, "Beyond Transformer Architecture: Griffin and Google RecurrentGemma",
// "Core Components of Griffin", 1. RG-LRU) is split into
//   unit = (batch row b, group of 128 output channels), tile = 64 tokens
//   (32 tokens when a head is 256 wide).
// For a tile, a warpgroup computes the width-4 Conv1D of the unit's input
// channels into a K-major bf16 operand in shared memory; one thread issues
// the gate contraction on the tensor core with the gate weights as the A
// operand (M = 128 output channels, MN-major, loaded by TMA) and the conv
// output as B (N = tokens), so that TMEM lane m holds channel m's two gate
// pre-activations along time. The same warpgroup then runs, per lane
// (channel), the sigmoid gates, the log-space decay, sqrt(1 - a^2), and the
// scan along time: the exact linear scan of S. De's thread ("we use linear
// scans"), carried across tiles by a decoupled look-back over per-tile
// (prod a, local h) aggregates and inclusive states in the workspace.
//
// Roles (320 threads, one CTA per SM, persistent):
//   warp 0      producer: claims tiles (per-unit counters, stealing from other
//               units once its own is done), TMA of x tiles and gate weights;
//   warp 1      TMEM owner and tcgen05.mma issuer;
//   warps 2-5   warpgroup 0, even jobs of this CTA;  warps 6-9 warpgroup 1, odd.
// Tiles of a unit are claimed in time order by running CTAs only, so every
// look-back waits on a tile that a running CTA owns. Every wait is bounded:
// on expiry the kernel records RGLRU_ERR_TIMEOUT, raises an abort flag that
// all waits observe, drains what it issued and returns.
#include <cudaTypedefs.h>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_primitives.cuh"

namespace rglru {
namespace {

using namespace tc;

constexpr int kM = 128;         // output channels per unit (MMA M, TMEM lanes)
constexpr int kJQ = 4;          // job ring depth
constexpr int kThreads = 320;
constexpr uint64_t kWaitNs = 2000000000ull;   // bound of any wait
constexpr uint64_t kDrainNs = 200000000ull;   // bound of the drain after an abort
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcParams {
  const __nv_bfloat16 *conv_w, *b_a, *b_x;
  const float *Lambda, *h0;
  const __nv_bfloat16 *conv_state_in;
  __nv_bfloat16 *y;
  float *h_T;
  __nv_bfloat16 *conv_state_out;
  int B, T, D, H, bw;
  int n_cg, n_units, n_tiles;
  int *counters, *abort_flag, *flags;
  float *aggA, *aggH, *incH;
  int *dev_status;
};

template <int K, int N, int NX>
struct Cfg {
  static constexpr int kXRows = N + 3;
  static constexpr int kXBytes = ((kXRows * K * 2) + 1023) / 1024 * 1024;
  static constexpr int kABytes = K * 256;          // one gate: 2 M-blocks x K rows x 128 B
  static constexpr int kBBytes = N * K * 2;        // one slot
  static constexpr int kOffA = 0;
  static constexpr int kOffX = 2 * kABytes;
  static constexpr int kOffB = kOffX + NX * kXBytes;
  static constexpr int kOffBar = kOffB + 2 * kBBytes;
  // barriers: job_full[JQ], job_empty[JQ], x_full[NX], x_empty[NX], w_full, b_full[2], acc_full[2]
  static constexpr int kNumBars = 2 * kJQ + 2 * NX + 1 + 2 + 2;
  static constexpr int kOffJobs = (kOffBar + kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kOffMisc = kOffJobs + kJQ * 16;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack
  // TMEM per slot: z_a (N columns), z_x (N), u (N); two slots.
  static constexpr int kSlotCols = 3 * N;
  static constexpr int kTmemCols = (2 * kSlotCols <= 128) ? 128 : (2 * kSlotCols <= 256 ? 256 : 512);
  static constexpr int kChunks = N / 32;   // conv: 32-token chunks
  static constexpr int kEChunks = N / 16;  // epilogue: 16-token chunks
  static_assert(N % 32 == 0 && K % 128 == 0, "tile shape");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(2 * kSlotCols <= 512, "TMEM allocation");
};

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

// Per element, from the gate pre-activations za, zx (bias included), the conv
// output u and nc2 = -c * softplus(-Lambda) * log2(e):
//   r = sigmoid(za) = sqrt_r^2 with sqrt_r = (1 + e^-za)^(-1/2),
//   i = sigmoid(zx) = (1 + tanh(zx / 2)) / 2,
//   log2 a = nc2 * r,  a = 2^(log2 a),
//   1 - a^2 = -expm1(2 ln a): a series in v = 2 ln a near a = 1, else 1 - a*a,
//   beta = sqrt(1 - a^2) * i * u.
__device__ __forceinline__ void gate_decay(float za, float zx, float u, float nc2, float &a,
                                           float &beta, float &la2) {
  const float e = ex2_approx(-za * kLog2e);
  const float q = rsqrt_approx(1.0f + e);
  const float r = q * q;
  const float ig = fmaf(0.5f, tanh_approx(0.5f * zx), 0.5f);
  la2 = nc2 * r;
  a = ex2_approx(la2);
  const float v = la2 * (2.0f * kLn2);
  // expm1(v) / v = 1 + v/2 + v^2/6 + v^3/24 + v^4/120 + v^5/720 (|v| <= 1/4)
  float p = fmaf(v, 1.0f / 720.0f, 1.0f / 120.0f);
  p = fmaf(v, p, 1.0f / 24.0f);
  p = fmaf(v, p, 1.0f / 6.0f);
  p = fmaf(v, p, 0.5f);
  p = fmaf(v, p, 1.0f);
  const float om = (v > -0.25f) ? (-v * p) : fmaf(-a, a, 1.0f);
  beta = sqrt_approx(om) * ig * u;
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ void raise_abort(const TcParams &p, volatile int *cta_abort, int code) {
  if (p.dev_status) atomicCAS(p.dev_status, 0, code);
  atomicExch(p.abort_flag, 1);
  *cta_abort = 1;
}

// Leader-side poll of a tile flag: returns the flag (1 aggregate, 2 inclusive),
// or -1 when another block aborted, or -2 on timeout.
__device__ int poll_flag(const int *flag, const int *gabort, volatile int *cta_abort) {
  int v = ld_acquire(flag);
  if (v) return v;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(40);
    v = ld_acquire(flag);
    if (v) return v;
    if (*cta_abort || *(volatile const int *)gabort) return -1;
    if (globaltimer_ns() - t0 > kWaitNs) return -2;
  }
}

template <int K, int N, int NX>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wa,
              const __grid_constant__ CUtensorMap tmap_wx, const TcParams p) {
  using C = Cfg<K, N, NX>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char *sA = sm + C::kOffA;
  unsigned char *sX = sm + C::kOffX;
  unsigned char *sB = sm + C::kOffB;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
  uint64_t *job_full = bars;
  uint64_t *job_empty = bars + kJQ;
  uint64_t *x_full = bars + 2 * kJQ;
  uint64_t *x_empty = x_full + NX;
  uint64_t *w_full = x_empty + NX;
  uint64_t *b_full = w_full + 1;
  uint64_t *acc_full = b_full + 2;
  int4 *jobs = reinterpret_cast<int4 *>(sm + C::kOffJobs);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::kOffMisc);
  volatile int *cta_abort = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 4);
  volatile int *bcast = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 8);  // [2]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- set-up: barriers, zero weight tiles (block-diagonal zeros), TMEM ----
  if (tid == 0) {
    for (int i = 0; i < kJQ; ++i) {
      mbar_init(&job_full[i], 1);
      mbar_init(&job_empty[i], 2);
    }
    for (int i = 0; i < NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
    }
    mbar_init(w_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&acc_full[i], 1);
    }
    *cta_abort = 0;
    bcast[0] = 0;
    bcast[1] = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_wa);
    prefetch_tmap(&tmap_wx);
  }
  {
    uint4 *a4 = reinterpret_cast<uint4 *>(sA);
    for (int i = tid; i < 2 * C::kABytes / 16; i += kThreads) a4[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int R = p.bw <= 128 ? p.bw : 256;           // weight rows per TMA box

  if (warp == 0) {
    // =============================== producer ===============================
    if (lane == 0) {
      int unit = blockIdx.x % p.n_units, scanned = 0, w_unit = -1;
      int i = 0, last_x_job = -1;
      bool ok = true;
      for (;; ++i) {
        int tile = -1;
        while (unit >= 0) {
          const int t = atomicAdd(&p.counters[unit], 1);
          if (t < p.n_tiles) {
            tile = t;
            break;
          }
          if (++scanned >= p.n_units) unit = -1;
          else unit = (unit + 1) % p.n_units;
        }
        if (*cta_abort) unit = -1;
        const int js = i % kJQ;
        if (!mbar_wait(&job_empty[js], ((i / kJQ) & 1) ^ 1, cta_abort, kWaitNs)) {
          if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
          ok = false;
          break;
        }
        const int reload = (unit >= 0 && unit != w_unit) ? 1 : 0;
        jobs[js] = make_int4(unit, tile, reload, 0);
        mbar_arrive(&job_full[js]);
        if (unit < 0) {
          const int j2 = (i + 1) % kJQ;
          if (mbar_wait(&job_empty[j2], (((i + 1) / kJQ) & 1) ^ 1, cta_abort, kWaitNs)) {
            jobs[j2] = make_int4(-1, -1, 0, 0);
            mbar_arrive(&job_full[j2]);
          }
          break;
        }
        const int b = unit / p.n_cg, cg = unit % p.n_cg;
        if (reload) {
          if (i > 0 && !mbar_wait(&job_empty[(i - 1) % kJQ], ((i - 1) / kJQ) & 1, cta_abort,
                                  kWaitNs)) {
            if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(w_full, 2u * 2u * static_cast<uint32_t>(R) * 128u);
          for (int g = 0; g < 2; ++g) {
            const CUtensorMap *tm = g == 0 ? &tmap_wa : &tmap_wx;
            unsigned char *dst = sA + g * C::kABytes;
            if (p.bw == 64) {
              for (int hh = 0; hh < 2; ++hh)
                tma_load_2d(dst + hh * (K * 128) + hh * 64 * 128, tm, w_full, 0,
                            (cg * 2 + hh) * 64);
            } else if (p.bw == 128) {
              for (int ma = 0; ma < 2; ++ma)
                tma_load_2d(dst + ma * (K * 128), tm, w_full, 64 * ma, cg * 128);
            } else {
              for (int ma = 0; ma < 2; ++ma)
                tma_load_2d(dst + ma * (K * 128), tm, w_full, (cg & 1) * 128 + 64 * ma,
                            (cg >> 1) * 256);
            }
          }
          w_unit = unit;
        }
        const int xb = i % NX;
        if (!mbar_wait(&x_empty[xb], ((i / NX) & 1) ^ 1, cta_abort, kWaitNs)) {
          if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
          ok = false;
          break;
        }
        const int kbase = p.bw <= 128 ? cg * kM : (cg >> 1) * 256;
        mbar_arrive_expect_tx(&x_full[xb], static_cast<uint32_t>(C::kXRows * K * 2));
        tma_load_3d(sX + xb * C::kXBytes, &tmap_x, &x_full[xb], kbase, tile * N - 3, b);
        last_x_job = i;
      }
      if (!ok || *cta_abort) {
        // drain: let every TMA this thread issued land before the CTA exits
        for (int j = last_x_job; j >= 0 && j > last_x_job - NX; --j)
          mbar_wait_drain(&x_full[j % NX], (j / NX) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kM, N, true, false);
      const uint32_t a0 = smem_u32(sA), a1 = smem_u32(sA + C::kABytes);
      uint32_t w_phase = 0;
      int last_commit = -1;
      for (int i = 0;; ++i) {
        const int js = i % kJQ;
        if (!mbar_wait(&job_full[js], (i / kJQ) & 1, cta_abort, kWaitNs)) {
          if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
          break;
        }
        const int4 job = jobs[js];
        if (job.x < 0) break;
        if (job.z) {
          if (!mbar_wait(w_full, w_phase, cta_abort, kWaitNs)) {
            if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
            break;
          }
          w_phase ^= 1;
        }
        const int s = i & 1;
        if (!mbar_wait(&b_full[s], (i >> 1) & 1, cta_abort, kWaitNs)) {
          if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t bs = smem_u32(sB + s * C::kBBytes);
        const uint32_t d_a = tmem_base + static_cast<uint32_t>(s * C::kSlotCols);
        const uint32_t d_x = d_a + N;
#pragma unroll
        for (int ks = 0; ks < K / 16; ++ks) {
          const uint64_t bd = sdesc_sw128(bs + (ks >> 2) * (N * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t ada = sdesc_sw128(a0 + ks * 16 * 128, K * 128, 1024);
          const uint64_t adx = sdesc_sw128(a1 + ks * 16 * 128, K * 128, 1024);
          mma_bf16(d_a, ada, bd, idesc, ks > 0 ? 1u : 0u);
          mma_bf16(d_x, adx, bd, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&acc_full[s]);
        last_commit = i;
        mbar_arrive(&job_empty[js]);
      }
      if (*cta_abort && last_commit >= 0)
        mbar_wait_drain(&acc_full[last_commit & 1], (last_commit >> 1) & 1, kDrainNs);
    }
  } else {
    // ============================== warpgroups ==============================
    const int wg = (warp - 2) >> 2;               // 0 or 1
    const int m = (warp & 3) * 32 + lane;         // TMEM lane == output channel in unit
    const bool leader = (warp == 2 + 4 * wg) && lane == 0;
    const int bar_id = 1 + wg;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(wg * C::kSlotCols);
    unsigned char *bslot = sB + wg * C::kBBytes;
    constexpr int KC = K / kM;                    // conv channels per thread (1 or 2)
    int cur_unit = -1;
    float cw[KC][4];
    float ba = 0.f, bx = 0.f, nc2 = 0.f;
    int own_kk = 0;

    for (int i = wg;; i += 2) {
      const int js = i % kJQ;
      if (!mbar_wait(&job_full[js], (i / kJQ) & 1, cta_abort, kWaitNs)) {
        if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
        break;
      }
      const int4 job = jobs[js];
      const int unit = job.x, tile = job.y;
      if (unit < 0) break;
      const int b = unit / p.n_cg, cg = unit % p.n_cg;
      const int c = cg * kM + m;                  // own output channel
      const int kbase = p.bw <= 128 ? cg * kM : (cg >> 1) * 256;
      if (unit != cur_unit) {
        cur_unit = unit;
        own_kk = p.bw <= 128 ? 0 : (cg & 1);
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
          const int ch = kbase + kk * kM + m;
#pragma unroll
          for (int tap = 0; tap < 4; ++tap) cw[kk][tap] = bf2f(p.conv_w[tap * p.D + ch]);
        }
        ba = bf2f(p.b_a[c]);
        bx = bf2f(p.b_x[c]);
        nc2 = -kDecayC * softplus_f32(-p.Lambda[c]) * kLog2e;
      }
      const int n0 = tile * N;
      const int nvalid = min(N, p.T - n0);
      const bool last_tile = (tile == p.n_tiles - 1);

      // ---- Conv1D into the B operand (and own channel's u in registers) ----
      const int xb = i % NX;
      if (!mbar_wait(&x_full[xb], (i / NX) & 1, cta_abort, kWaitNs)) {
        if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
        break;
      }
      const __nv_bfloat16 *xs = reinterpret_cast<const __nv_bfloat16 *>(sX + xb * C::kXBytes);
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        const int k = kk * kM + m;                // index within the K range
        float xm3 = bf2f(xs[0 * K + k]), xm2 = bf2f(xs[1 * K + k]), xm1 = bf2f(xs[2 * K + k]);
        if (tile == 0 && p.conv_state_in != nullptr) {
          const __nv_bfloat16 *cs = p.conv_state_in + static_cast<size_t>(b) * 3 * p.D + kbase + k;
          xm3 = bf2f(cs[0]);
          xm2 = bf2f(cs[p.D]);
          xm1 = bf2f(cs[2 * p.D]);
        }
        const bool own = (kk == own_kk);          // uniform across the warpgroup
        // byte offsets of (row n, channel k) in the swizzled operand depend on n % 8 only,
        // besides the n * 128 row term
        uint32_t colo[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) colo[r] = kmajor_sw128_offset(r, k, N) - r * 128;
#pragma unroll
        for (int ch = 0; ch < C::kEChunks; ++ch) {
          float uc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = ch * 16 + j;
            const float xv = bf2f(xs[(n + 3) * K + k]);
            const float u =
                fmaf(cw[kk][3], xv, fmaf(cw[kk][2], xm1, fmaf(cw[kk][1], xm2, cw[kk][0] * xm3)));
            xm3 = xm2;
            xm2 = xm1;
            xm1 = xv;
            *reinterpret_cast<__nv_bfloat16 *>(bslot + colo[n & 7] + n * 128) =
                __float2bfloat16_rn(u);
            uc[j] = u;
            if (own && last_tile && n == nvalid - 1 && p.conv_state_out != nullptr) {
              __nv_bfloat16 *co = p.conv_state_out + static_cast<size_t>(b) * 3 * p.D + c;
              co[0] = __float2bfloat16_rn(xm3);
              co[p.D] = __float2bfloat16_rn(xm2);
              co[2 * p.D] = __float2bfloat16_rn(xm1);
            }
          }
          if (own) tmem_st16(t_lane + 2 * N + ch * 16, uc);   // own channel's u for beta
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      named_bar_sync(bar_id, 128);
      if (leader) {
        mbar_arrive(&x_empty[xb]);
        mbar_arrive(&b_full[wg]);
      }

      // ---- gates, decay, local scan (pass 1) ----
      if (!mbar_wait(&acc_full[wg], (i >> 1) & 1, cta_abort, kWaitNs)) {
        if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      float Hl = 0.f, S = 0.f;
#pragma unroll
      for (int ch = 0; ch < C::kEChunks; ++ch) {
        float za[16], zx[16], uu[16];
        tmem_ld16(t_lane + ch * 16, za);
        tmem_ld16(t_lane + N + ch * 16, zx);
        tmem_ld16(t_lane + 2 * N + ch * 16, uu);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = ch * 16 + j;
          float a, beta, la2;
          gate_decay(za[j] + ba, zx[j] + bx, uu[j], nc2, a, beta, la2);
          if (n >= nvalid) {
            a = 1.f;
            beta = 0.f;
            la2 = 0.f;
          }
          Hl = fmaf(a, Hl, beta);
          S += la2;
          za[j] = a;
          zx[j] = beta;
        }
        tmem_st16(t_lane + ch * 16, za);
        tmem_st16(t_lane + N + ch * 16, zx);
      }
      tmem_wait_st();
      const float A = ex2_approx(S);

      // ---- carry across tiles: decoupled look-back ----
      const size_t tix = static_cast<size_t>(unit) * p.n_tiles + tile;
      float h_in = 0.f;
      if (tile == 0) {
        if (p.h0 != nullptr) h_in = p.h0[static_cast<size_t>(b) * p.D + c];
      } else {
        __stcg(p.aggA + tix * kM + m, A);
        __stcg(p.aggH + tix * kM + m, Hl);
        __threadfence();
        named_bar_sync(bar_id, 128);
        if (leader) st_release(p.flags + tix, 1);
        float mult = 1.f, add = 0.f;
        int jt = tile - 1;
        for (;;) {
          if (leader) {
            int f = poll_flag(p.flags + static_cast<size_t>(unit) * p.n_tiles + jt, p.abort_flag,
                              cta_abort);
            if (f == -2) {
              raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT);
              f = -1;
            }
            bcast[wg] = f;
          }
          named_bar_sync(bar_id, 128);
          const int f = bcast[wg];
          named_bar_sync(bar_id, 128);
          const size_t jix = (static_cast<size_t>(unit) * p.n_tiles + jt) * kM + m;
          if (f == 2) {
            h_in = fmaf(mult, __ldcg(p.incH + jix), add);
            break;
          }
          if (f != 1) {
            h_in = 0.f;
            break;
          }
          add = fmaf(mult, __ldcg(p.aggH + jix), add);
          mult *= __ldcg(p.aggA + jix);
          --jt;
        }
      }
      __stcg(p.incH + tix * kM + m, fmaf(A, h_in, Hl));
      __threadfence();
      named_bar_sync(bar_id, 128);
      if (leader) st_release(p.flags + tix, 2);

      // ---- final scan (pass 2): y_t = h_t ----
      float h = h_in;
      __nv_bfloat16 *yrow = p.y + (static_cast<size_t>(b) * p.T + n0) * p.D + c;
#pragma unroll
      for (int ch = 0; ch < C::kEChunks; ++ch) {
        float av[16], bv[16];
        tmem_ld16(t_lane + ch * 16, av);
        tmem_ld16(t_lane + N + ch * 16, bv);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = ch * 16 + j;
          h = fmaf(av[j], h, bv[j]);
          if (n < nvalid) yrow[static_cast<size_t>(n) * p.D] = __float2bfloat16_rn(h);
        }
      }
      if (last_tile && p.h_T != nullptr) p.h_T[static_cast<size_t>(b) * p.D + c] = h;
      tc_fence_before();
      named_bar_sync(bar_id, 128);
      if (leader) mbar_arrive(&job_empty[js]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ------------------------------------------------------------------ host --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

int tile_tokens(int bw) { return bw == 256 ? 32 : 64; }

struct TcLayout {
  int n_cg, n_units, n_tiles;
  size_t off_counters, off_abort, off_flags, off_aggA, off_aggH, off_incH, ints_bytes, total;
};

TcLayout tc_layout(int B, int T, int D, int H) {
  TcLayout L{};
  const int bw = D / H;
  L.n_cg = D / kM;
  L.n_units = B * L.n_cg;
  L.n_tiles = ceil_div(T, tile_tokens(bw));
  L.off_counters = 0;
  L.off_abort = static_cast<size_t>(L.n_units) * 4;
  L.off_flags = align_up(L.off_abort + 4, 16);
  L.ints_bytes = align_up(L.off_flags + static_cast<size_t>(L.n_units) * L.n_tiles * 4, 256);
  const size_t agg = align_up(static_cast<size_t>(L.n_units) * L.n_tiles * kM * 4, 256);
  L.off_aggA = L.ints_bytes;
  L.off_aggH = L.off_aggA + agg;
  L.off_incH = L.off_aggH + agg;
  L.total = L.off_incH + agg;
  return L;
}

template <int K, int N, int NX>
cudaError_t launch_tc_t(const FwdArgs &a, const TcLayout &L, void *ws, cudaStream_t st) {
  using C = Cfg<K, N, NX>;
  auto enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const int bw = a.D / a.H;
  CUtensorMap tx, twa, twx;
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.D), static_cast<cuuint64_t>(a.T),
                          static_cast<cuuint64_t>(a.B)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.D) * 2,
                             static_cast<cuuint64_t>(a.T) * a.D * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(K), static_cast<cuuint32_t>(N + 3), 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.x), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int R = bw <= 128 ? bw : 256;
  for (int g = 0; g < 2; ++g) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(bw), static_cast<cuuint64_t>(a.H) * bw};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(bw) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(R)};
    cuuint32_t es[2] = {1, 1};
    if (enc(g == 0 ? &twa : &twx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void *>(g == 0 ? a.W_a : a.W_x), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  unsigned char *w = static_cast<unsigned char *>(ws);
  TcParams p;
  p.conv_w = static_cast<const __nv_bfloat16 *>(a.conv_w);
  p.b_a = static_cast<const __nv_bfloat16 *>(a.b_a);
  p.b_x = static_cast<const __nv_bfloat16 *>(a.b_x);
  p.Lambda = a.Lambda;
  p.h0 = a.h0;
  p.conv_state_in = static_cast<const __nv_bfloat16 *>(a.conv_state_in);
  p.y = static_cast<__nv_bfloat16 *>(a.y);
  p.h_T = a.h_T;
  p.conv_state_out = static_cast<__nv_bfloat16 *>(a.conv_state_out);
  p.B = a.B;
  p.T = a.T;
  p.D = a.D;
  p.H = a.H;
  p.bw = bw;
  p.n_cg = L.n_cg;
  p.n_units = L.n_units;
  p.n_tiles = L.n_tiles;
  p.counters = reinterpret_cast<int *>(w + L.off_counters);
  p.abort_flag = reinterpret_cast<int *>(w + L.off_abort);
  p.flags = reinterpret_cast<int *>(w + L.off_flags);
  p.aggA = reinterpret_cast<float *>(w + L.off_aggA);
  p.aggH = reinterpret_cast<float *>(w + L.off_aggH);
  p.incH = reinterpret_cast<float *>(w + L.off_incH);
  p.dev_status = a.dev_status;

  cudaError_t e = cudaMemsetAsync(ws, 0, L.ints_bytes, st);
  if (e != cudaSuccess) return e;
  auto kern = fwd_tc_kernel<K, N, NX>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long jobs = static_cast<long>(L.n_units) * L.n_tiles;
  const int grid = static_cast<int>(jobs < sms ? jobs : sms);
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(tx, twa, twx, p);
  return cudaGetLastError();
}

}  // namespace

bool tc_supported(int B, int T, int D, int H, int io) {
  if (io != RGLRU_IO_BF16) return false;
  if (D % kM != 0 || D % H != 0) return false;
  const int bw = D / H;
  return bw == 64 || bw == 128 || bw == 256;
}

size_t tc_workspace_bytes(int B, int T, int D, int H) { return tc_layout(B, T, D, H).total; }

cudaError_t launch_fwd_tc(const FwdArgs &a, void *ws, cudaStream_t st) {
  const int bw = a.D / a.H;
  const TcLayout L = tc_layout(a.B, a.T, a.D, a.H);
  if (bw == 256) return launch_tc_t<256, 32, 2>(a, L, ws, st);
  return launch_tc_t<128, 64, 3>(a, L, ws, st);
}

}  // namespace rglru
