// One RG-LRU decode step for B sequences on the tensor core (sm_100a), bf16 I/O.
//
// The layer at one time step ("Griffin: Mixing Gated Linear Recurrences with
// Local Attention for Efficient Language Models", section "Model
// Architecture"; the fixed-size state that makes decoding cheap is the point
// of "Beyond Transformer Architecture: Griffin and Google RecurrentGemma",
// "Core Components of Griffin", 1. RG-LRU):
//   u = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t      (three past inputs in a ring)
//   [z_a | z_x] = u W (block-diagonal), gates, a, beta as in the forward
//   h <- a h + beta,  y_t = h,  ring slot pos % 3 <- x_t
// Jobs are (group of 128 output channels, tile of N = 16 batch rows). The gate
// contraction runs on tcgen05 with the gate weights as A (M = 128 channels) and
// the conv output as B (N = rows), so TMEM lane m holds channel m's gates for
// the tile's rows; the epilogue updates h in place lane = channel, which keeps
// its global accesses coalesced. Rows never interact, so CTAs take balanced
// contiguous ranges of jobs and nothing waits on another CTA.
//
// Roles: warp 0 posts the CTA's jobs and loads by TMA the gate weights and,
// two jobs ahead, each job's inputs (x_t and the three ring slots of its rows
// and channels); warp 1 owns TMEM and issues the MMAs; warps 2-5 compute the
// Conv1D from shared memory into the bf16 B operand and an fp32 u tile; two
// epilogue warpgroups take the jobs alternately and load their rows' h before
// waiting for the MMA.
//
// Heads 256 wide run as CTA pairs (a cluster of 2): the two 128-channel units
// of a head take the same row tiles; each CTA loads x_t and the ring slots of
// its own 128 channels only, computes their Conv1D, and sends its half of the
// MMA's B operand (all 256 input channels) to the partner by a bulk copy that
// completes on the partner's barrier; the MMA releases a B slot to both CTAs.
// Each CTA is then the only reader of its channels' ring slot and rewrites it
// with x_t itself, so a step is one launch for every head width.
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tc_gates.cuh"
#include "tc_pair.cuh"
#include "tc_primitives.cuh"

namespace rglru {
namespace {

using namespace tc;
using namespace gates;

constexpr int kM = 128;
constexpr int kJQ = 8;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;

struct DecTcParams {
  const __nv_bfloat16 *conv_w, *b_a, *b_x;
  const __nv_bfloat16 *W_a, *W_x;            // (H, bw, bw): read directly when A is in TMEM
  const float *Lambda;
  __nv_bfloat16 *ring;
  const __nv_bfloat16 *x_t;
  float *h;
  __nv_bfloat16 *y_t;
  int B, D, H, bw, pos;
  int n_cg, n_tiles, n_jobs;
  int write_ring;                  // 1: this kernel rewrites ring slot pos % 3
};

template <int K, int N>
struct DCfg {
  static constexpr int NE = 2;                     // epilogue warpgroups
  static constexpr int kThreads = 64 + 128 + NE * 128;
  // Gate weights (the MMA's A operand), TMA-loaded into shared memory at each
  // change of unit: the MMA reads them there for K = 128; for K = 256 the conv
  // warpgroup copies them into TMEM once per unit, where the tensor core would
  // otherwise re-read 128 KB of shared memory for every 16-row job
  static constexpr bool kATmem = (K == 256);
  static constexpr int kABytes = K * 256;          // one gate: 2 M-blocks x K rows x 128 B
  // 256-wide heads run as CTA pairs (a cluster of 2, one per 128-channel unit of
  // the head, on the same rows): each CTA loads and convolves only its own 128
  // channels and sends its half of the B operand to the partner
  static constexpr bool kPair = (K == 256);
  static constexpr int kXK = kPair ? kM : K;       // channels of an input tile
  static constexpr int kInBytes = N * kXK * 2;     // one input tile: N rows x kXK channels, bf16
  static constexpr int kXBytes = 4 * kInBytes;     // x_t and ring slots pos, pos+1, pos+2 (mod 3)
  static constexpr int kNX = kPair ? 3 : 2;        // input slots
  static constexpr int kBBytes = N * K * 2;
  static constexpr int kUBytes = N * kM * 4;
  // B operand and u tile slots (a pair's third slot absorbs the partner's lag)
  static constexpr int kNS = kPair ? 3 : 2;
  static constexpr int kNT = NE + 1;
  static constexpr int kOffA = 0;
  static constexpr int kOffX = 2 * kABytes;
  static constexpr int kOffB = kOffX + kNX * kXBytes;
  static constexpr int kOffU = kOffB + kNS * kBBytes;
  static constexpr int kOffBar = kOffU + kNS * kUBytes;
  // job_full[JQ], job_empty[JQ], x_full[NX], x_empty[NX], w_full, w_free,
  // b_full[NS], b_empty[NS], u_empty[NS], acc_full[NT], tmem_empty[NT], a_ready
  static constexpr int kNumBars = 2 * kJQ + 2 * kNX + 2 + 3 * kNS + 2 * kNT + 1;
  static constexpr int kOffJobs = (kOffBar + kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kOffMisc = kOffJobs + kJQ * 16;
  // the dynamic shared memory base is declared 1024-byte aligned (checked)
  static constexpr int kSmemBytes = kOffMisc + 64;
  static constexpr int kSlotCols = 2 * N;
  static constexpr int kACol = kNT * kSlotCols;             // TMEM A: gate a, then gate x
  static constexpr int kUsedCols = kACol + (kATmem ? K : 0);
  static constexpr int kTmemCols = kUsedCols <= 128 ? 128 : (kUsedCols <= 256 ? 256 : 512);
  static_assert(kUsedCols <= 512, "TMEM allocation");
  static constexpr int NQ = kXK / 4;               // conv: channel quads
  static constexpr int SEG = N * NQ / 128;         // conv: rows per thread
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(N % 16 == 0 && (N * NQ) % 128 == 0 && SEG % 4 == 0, "conv mapping");
};

// One 16-bit shared-memory load (zero-extended).
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
  return v;
}

// Offset (bytes) of (own channel c, 4-row block jb) in the fp32 u tile:
// channel-major rows of N floats whose 16-byte blocks are XOR-permuted so that
// any 8 consecutive channels (a quarter warp of epilogue readers) hit distinct
// banks: with 8 or more blocks per row by (c % 8) ^ (c / 8 % 8); with 4 blocks
// (two rows per 128 bytes) by (c / 2) % 4.
template <int N>
__device__ __forceinline__ uint32_t u_off(int c, int jb) {
  static_assert(N == 16 || N >= 32, "u tile rows of 4 or of at least 8 blocks");
  const int perm = N == 16 ? ((c >> 1) & 3) : ((c & 7) ^ ((c >> 3) & 7));
  return static_cast<uint32_t>(c * (N * 4) + ((jb ^ perm) << 4));
}

// Conv1D of N rows x kXK channels from the input tile in shared memory
// (row-major [N][kXK] per array: x_t, then the ring slots holding x_{t-3},
// x_{t-2}, x_{t-1}). Thread t covers channel quad q (4 channels) and SEG
// consecutive rows. Writes the bf16 K-major B operand (128-byte swizzle) at K
// rows koff + channel, the fp32 u of the own channels (channel-major, see
// u_off) and, when asked, the ring update of the own channels.
template <int K, int N>
__device__ __forceinline__ void dec_conv(const DecTcParams &p, const unsigned char *__restrict__ xin,
                                         unsigned char *__restrict__ bt,
                                         unsigned char *__restrict__ ut, int kbase, int own_lo,
                                         int koff, int r0, int t, const float2 (&w)[4][2]) {
  using C = DCfg<K, N>;
  constexpr int NQ = C::NQ, SEG = C::SEG, XK = C::kXK;
  const int qd = t % NQ, sg = t / NQ;
  const int kq = qd * 4, nb = sg * SEG;
  const bool own = (kq >= own_lo) && (kq < own_lo + kM);
  const int chq = kbase + kq;
  const int s0 = p.pos % 3;
  const int kk = koff + kq;                        // K row of the quad in the B operand
  const unsigned char *xq = xin + kq * 2;          // + array * kInBytes + row * XK * 2
  unsigned char *bq = bt + (kk >> 6) * N * 128 + ((kk & 7) << 1);
  const int chunk = (kk & 63) >> 3;
#pragma unroll
  for (int j0 = 0; j0 < SEG; j0 += 4) {
    float uacc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = nb + j0 + j;
      const uint2 xv = *reinterpret_cast<const uint2 *>(xq + n * XK * 2);
      const uint2 r0v = *reinterpret_cast<const uint2 *>(xq + C::kInBytes + n * XK * 2);
      const uint2 r1v = *reinterpret_cast<const uint2 *>(xq + 2 * C::kInBytes + n * XK * 2);
      const uint2 r2v = *reinterpret_cast<const uint2 *>(xq + 3 * C::kInBytes + n * XK * 2);
      float2 u[2];
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const uint32_t a0 = pp ? r0v.y : r0v.x, a1 = pp ? r1v.y : r1v.x;
        const uint32_t a2 = pp ? r2v.y : r2v.x, a3 = pp ? xv.y : xv.x;
        float2 acc = __fmul2_rn(w[0][pp], bf2_to_f2(a0));
        acc = __ffma2_rn(w[1][pp], bf2_to_f2(a1), acc);
        acc = __ffma2_rn(w[2][pp], bf2_to_f2(a2), acc);
        u[pp] = __ffma2_rn(w[3][pp], bf2_to_f2(a3), acc);
      }
      *reinterpret_cast<uint2 *>(bq + n * 128 + (((chunk ^ n) & 7) << 4)) =
          make_uint2(f2_to_bf2(u[0]), f2_to_bf2(u[1]));
      uacc[0][j] = u[0].x;
      uacc[1][j] = u[0].y;
      uacc[2][j] = u[1].x;
      uacc[3][j] = u[1].y;
      const int row = r0 + n;
      if (p.write_ring && own && row < p.B)
        *reinterpret_cast<uint2 *>(p.ring + static_cast<size_t>(row) * 3 * p.D +
                                   static_cast<size_t>(s0) * p.D + chq) = xv;
    }
    if (own) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<float4 *>(ut + u_off<N>(kq - own_lo + k, (nb + j0) >> 2)) =
            make_float4(uacc[k][0], uacc[k][1], uacc[k][2], uacc[k][3]);
    }
  }
}

template <int K, int N>
__global__ void __launch_bounds__(DCfg<K, N>::kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_wa,
                 const __grid_constant__ CUtensorMap tmap_wx,
                 const __grid_constant__ CUtensorMap tmap_xt,
                 const __grid_constant__ CUtensorMap tmap_ring, const DecTcParams p) {
  using C = DCfg<K, N>;
  constexpr int NS = C::kNS, NT = C::kNT, NE = C::NE, NX = C::kNX;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) return;   // the layout needs the declared alignment
  unsigned char *sm = smem_raw;
  unsigned char *sA = sm + C::kOffA;
  unsigned char *sX = sm + C::kOffX;
  unsigned char *sB = sm + C::kOffB;
  unsigned char *sU = sm + C::kOffU;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
  uint64_t *job_full = bars;
  uint64_t *job_empty = job_full + kJQ;
  uint64_t *x_full = job_empty + kJQ;
  uint64_t *x_empty = x_full + NX;
  uint64_t *w_full = x_empty + NX;
  uint64_t *w_free = w_full + 1;
  uint64_t *b_full = w_free + 1;
  uint64_t *b_empty = b_full + NS;
  uint64_t *u_empty = b_empty + NS;
  uint64_t *acc_full = u_empty + NS;
  uint64_t *tmem_empty = acc_full + NT;
  uint64_t *a_ready = tmem_empty + NT;              // conv warpgroup wrote TMEM weights -> MMA
  int4 *jobs = reinterpret_cast<int4 *>(sm + C::kOffJobs);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::kOffMisc);
  volatile int *cta_abort = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr bool kPair = C::kPair;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  // this CTA's (pair's) contiguous, balanced range of work items: jobs (unit *
  // n_tiles + tile), or for CTA pairs (head * n_tiles + tile), the CTA of rank r
  // taking unit 2 head + r
  const int n_items = kPair ? p.n_jobs / 2 : p.n_jobs;
  const int n_grp = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int grp = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int j_begin = static_cast<int>(static_cast<long>(n_items) * grp / n_grp);
  const int j_end = static_cast<int>(static_cast<long>(n_items) * (grp + 1) / n_grp);

  if (tid == 0) {
    for (int i = 0; i < kJQ; ++i) {
      mbar_init(&job_full[i], 1);
      mbar_init(&job_empty[i], 9);                  // 4 conv warps, MMA, 4 epilogue warps
    }
    for (int i = 0; i < NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 4);                    // 4 conv warps
    }
    mbar_init(w_full, 1);
    mbar_init(w_free, C::kATmem ? 4 : 1);          // the conv warps' TMEM copy, or the MMA
    for (int i = 0; i < NS; ++i) {
      // 4 conv warps; for a pair each also expects the bytes of the partner's
      // matching warp (bulk copies of its half of the B operand)
      mbar_init(&b_full[i], 4);
      mbar_init(&b_empty[i], kPair ? 2 : 1);        // MMA commit (of each CTA of a pair)
      mbar_init(&u_empty[i], 4);
    }
    for (int i = 0; i < NT; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&tmem_empty[i], 4);
    }
    mbar_init(a_ready, 4);                          // 4 conv warps
    *cta_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_wa);
    prefetch_tmap(&tmap_wx);
    prefetch_tmap(&tmap_xt);
    prefetch_tmap(&tmap_ring);
  }
  if (!C::kATmem) {
    // block-diagonal zeros of 64-wide heads (the TMA fills 256-wide heads' tiles whole)
    uint4 *a4 = reinterpret_cast<uint4 *>(sA);
    for (int i = tid; i < 2 * C::kABytes / 16; i += C::kThreads) a4[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // a pair's barriers are initialised before either CTA arrives on the other's
  if (kPair)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int R = p.bw <= 128 ? p.bw : 256;
  const uint32_t peer_abort =
      kPair ? mapa_shared(smem_u32(const_cast<int *>(cta_abort)), rank ^ 1u) : 0u;

#define RG_WAIT_OR_ABORT(bar, par)                        \
  if (!mbar_wait((bar), (par), cta_abort, kWaitNs)) {      \
    *cta_abort = 1;                                       \
    if (kPair) st_cluster_u32(peer_abort, 1u);            \
    break;                                                \
  }

  if (warp == 0) {
    // ============================== job poster ==============================
    if (lane == 0) {
      int w_unit = -1;
      uint32_t wfree_phase = 0;
      const int n = j_end - j_begin;
      int last_x_job = -1;
      for (int i = 0; i <= n + NE - 1; ++i) {
        const int js = i % kJQ;
        RG_WAIT_OR_ABORT(&job_empty[js], ((i / kJQ) & 1) ^ 1);
        if (i >= n) {                                // terminal jobs, one per epilogue warpgroup
          jobs[js] = make_int4(-1, -1, 0, 0);
          mbar_arrive(&job_full[js]);
          continue;
        }
        const int item = j_begin + i;
        const int unit = kPair ? 2 * (item / p.n_tiles) + static_cast<int>(rank) : item / p.n_tiles;
        const int tile = item % p.n_tiles;
        const int reload = unit != w_unit ? 1 : 0;
        jobs[js] = make_int4(unit, tile, reload, 0);
        mbar_arrive(&job_full[js]);
        const int cg = unit;
        if (reload) {
          if (i > 0) {
            RG_WAIT_OR_ABORT(w_free, wfree_phase);
            wfree_phase ^= 1;
          }
          mbar_arrive_expect_tx(w_full, 2u * 2u * static_cast<uint32_t>(R) * 128u);
          for (int g = 0; g < 2; ++g) {
            const CUtensorMap *tm = g == 0 ? &tmap_wa : &tmap_wx;
            unsigned char *dst = sA + g * C::kABytes;
            if (p.bw == 64) {
              for (int hh = 0; hh < 2; ++hh)
                tma_load_2d(dst + hh * (K * 128) + hh * 64 * 128, tm, w_full, 0, (cg * 2 + hh) * 64);
            } else if (p.bw == 128) {
              for (int ma = 0; ma < 2; ++ma)
                tma_load_2d(dst + ma * (K * 128), tm, w_full, 64 * ma, cg * 128);
            } else {
              for (int ma = 0; ma < 2; ++ma)
                tma_load_2d(dst + ma * (K * 128), tm, w_full, (cg & 1) * 128 + 64 * ma,
                            (cg >> 1) * 256);
            }
          }
        }
        if (reload) w_unit = unit;
        // the job's inputs: x_t rows, then ring slots pos % 3 (x_{t-3}),
        // (pos + 1) % 3 (x_{t-2}), (pos + 2) % 3 (x_{t-1}); rows past B read as zeros
        const int xb = i % NX;
        RG_WAIT_OR_ABORT(&x_empty[xb], ((i / NX) & 1) ^ 1);
        // input channels of the job: the unit's own 128 (CTA pairs, heads up to
        // 128 wide), else the head's 256
        const int kbase = (kPair || p.bw <= 128) ? cg * kM : (cg >> 1) * 256;
        unsigned char *dst = sX + xb * C::kXBytes;
        mbar_arrive_expect_tx(&x_full[xb], static_cast<uint32_t>(C::kXBytes));
        tma_load_2d(dst, &tmap_xt, &x_full[xb], kbase, tile * N);
        for (int q = 0; q < 3; ++q)
          tma_load_3d(dst + (q + 1) * C::kInBytes, &tmap_ring, &x_full[xb], kbase, (p.pos + q) % 3,
                      tile * N);
        last_x_job = i;
      }
      if (*cta_abort) {
        for (int j = last_x_job; j >= 0 && j > last_x_job - NX; --j)
          mbar_wait_drain(&x_full[j % NX], (j / NX) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    if (lane == 0) {
      // A from shared memory is MN-major (loaded by TMA); A from TMEM is K-major
      constexpr uint32_t idesc = idesc_bf16_f32(kM, N, !C::kATmem, false);
      const uint64_t ada0 = sdesc_sw128(smem_u32(sA), K * 128, 1024);
      const uint64_t adx0 = sdesc_sw128(smem_u32(sA + C::kABytes), K * 128, 1024);
      const uint32_t ta_a = tmem_base + static_cast<uint32_t>(C::kACol);
      const uint32_t ta_x = ta_a + static_cast<uint32_t>(K / 2);
      uint32_t w_phase = 0;
      int last_commit = -1;
      for (int i = 0;; ++i) {
        const int js = i % kJQ;
        RG_WAIT_OR_ABORT(&job_full[js], (i / kJQ) & 1);
        const int4 job = jobs[js];
        if (job.x < 0) break;
        if (job.z) {
          if (C::kATmem) {
            // the conv warpgroup has written this unit's weights into TMEM
            RG_WAIT_OR_ABORT(a_ready, w_phase);
          } else {
            if (last_commit >= 0) {
              const int lc = last_commit;
              RG_WAIT_OR_ABORT(&acc_full[lc % NT], (lc / NT) & 1);
              mbar_arrive(w_free);
            }
            RG_WAIT_OR_ABORT(w_full, w_phase);
          }
          w_phase ^= 1;
        }
        const int s = i % NS, ts = i % NT;
        RG_WAIT_OR_ABORT(&b_full[s], (i / NS) & 1);
        RG_WAIT_OR_ABORT(&tmem_empty[ts], ((i / NT) & 1) ^ 1);
        tc_fence_after();
        const uint32_t bs = smem_u32(sB + s * C::kBBytes);
        const uint32_t d_a = tmem_base + static_cast<uint32_t>(ts * C::kSlotCols);
        const uint32_t d_x = d_a + N;
        // descriptors of K step 0; a step advances the start addresses by a
        // constant (the address field holds address / 16, and shared-memory
        // addresses stay below 256 KB, so the additions never carry out of it)
        const uint64_t bd0 = sdesc_sw128(bs, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < K / 16; ++ks) {
          const uint64_t bd = bd0 + static_cast<uint64_t>(((ks >> 2) * (N * 128) + (ks & 3) * 32) >> 4);
          if (C::kATmem) {
            mma_bf16_ts(d_a, ta_a + static_cast<uint32_t>(ks * 8), bd, idesc, ks > 0 ? 1u : 0u);
            mma_bf16_ts(d_x, ta_x + static_cast<uint32_t>(ks * 8), bd, idesc, ks > 0 ? 1u : 0u);
          } else {
            const uint64_t astep = static_cast<uint64_t>((ks * 16 * 128) >> 4);
            mma_bf16(d_a, ada0 + astep, bd, idesc, ks > 0 ? 1u : 0u);
            mma_bf16(d_x, adx0 + astep, bd, idesc, ks > 0 ? 1u : 0u);
          }
        }
        mma_commit(&acc_full[ts]);
        // the B slot is free once the MMAs of both CTAs of a pair have read it
        if (kPair)
          mma_commit_multicast(&b_empty[s], 0x3);
        else
          mma_commit(&b_empty[s]);
        last_commit = i;
        mbar_arrive(&job_empty[js]);
      }
      if (*cta_abort && last_commit >= 0)
        mbar_wait_drain(&acc_full[last_commit % NT], (last_commit / NT) & 1, kDrainNs);
    }
  } else if (warp < 6) {
    // ============================== conv warpgroup ==============================
    const int wt = tid - 64;
    int cur_unit = -1;
    uint32_t wfull_phase = 0;
    float2 cwq[4][2];
    // CTA pairs: the partner's B slots and b_full barriers (shared::cluster), and
    // this warp's rows of the B operand (see dec_conv: SEG rows per warp)
    const uint32_t sB_peer = kPair ? mapa_shared(smem_u32(sB), rank ^ 1u) : 0u;
    const uint32_t bfull_peer = kPair ? mapa_shared(smem_u32(b_full), rank ^ 1u) : 0u;
    const uint32_t seg_off = static_cast<uint32_t>((wt >> 5) * C::SEG * 128);
    int i = 0;
    for (;; ++i) {
      const int js = i % kJQ;
      RG_WAIT_OR_ABORT(&job_full[js], (i / kJQ) & 1);
      const int4 job = jobs[js];
      const int unit = job.x, tile = job.y;
      if (unit < 0) break;
      const int cg = unit;
      // the input channels convolved here (the unit's own 128 for pairs and
      // heads up to 128 wide), the own ones among them, and their K rows in B
      const int kbase = (kPair || p.bw <= 128) ? cg * kM : (cg >> 1) * 256;
      const int own_lo = (kPair || p.bw <= 128) ? 0 : (cg & 1) * kM;
      const int koff = kPair ? (cg & 1) * kM : 0;
      if (unit != cur_unit) {
        cur_unit = unit;
        const int chq = kbase + (wt % C::NQ) * 4;
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
          const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.conv_w + tap * p.D + chq));
          cwq[tap][0] = bf2_to_f2(raw.x);
          cwq[tap][1] = bf2_to_f2(raw.y);
        }
        if (C::kATmem) {
          // This unit's gate weights into TMEM (the A operand): lane m (output
          // channel cg*128 + m) holds W[h][k][j] for k = 0..K-1, two per column,
          // copied from the TMA-loaded shared-memory tiles (128-byte swizzle,
          // MN-major: per 64-channel block ma, row k of 128 B, 16-byte chunk
          // (m % 64) / 8 stored at chunk ^ (k % 8); a warp's 32 channels read
          // 64 bytes of one row: no bank conflicts). Every MMA of earlier jobs
          // has read the old TMEM weights once the accumulator of job i-1 is
          // complete (MMAs complete in issue order).
          RG_WAIT_OR_ABORT(w_full, wfull_phase);
          wfull_phase ^= 1;
          if (i > 0) RG_WAIT_OR_ABORT(&acc_full[(i - 1) % NT], ((i - 1) / NT) & 1);
          const int qd = warp & 3;                  // this warp's TMEM lane quadrant
          const int m = qd * 32 + lane;             // output channel within the unit
          const uint32_t tq = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                              static_cast<uint32_t>(C::kACol);
          const uint32_t mcol = static_cast<uint32_t>((m >> 6) * (K * 128) + ((m & 7) << 1));
          const uint32_t mchunk = static_cast<uint32_t>((m & 63) >> 3);
#pragma unroll 1
          for (int g = 0; g < 2; ++g) {
            const uint32_t ag = smem_u32(sA + g * C::kABytes) + mcol;
#pragma unroll 1
            for (int cc = 0; cc < K / 64; ++cc) {
              uint32_t v[32];
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                const uint32_t k = static_cast<uint32_t>(cc * 64 + 2 * q);   // even: k % 8 = 2q % 8
                const uint32_t lo = lds_u16(ag + k * 128 + ((mchunk ^ (k & 7)) << 4));
                const uint32_t hi = lds_u16(ag + (k + 1) * 128 + ((mchunk ^ ((k + 1) & 7)) << 4));
                v[q] = lo | (hi << 16);
              }
              tmem_st32u(tq + static_cast<uint32_t>(g * (K / 2) + cc * 32), v);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(a_ready);
            mbar_arrive(w_free);                    // the shared-memory tiles may be reloaded
          }
        }
      }
      const int s = i % NS, xb = i % NX;
      RG_WAIT_OR_ABORT(&x_full[xb], (i / NX) & 1);
      RG_WAIT_OR_ABORT(&b_empty[s], ((i / NS) & 1) ^ 1);
      RG_WAIT_OR_ABORT(&u_empty[s], ((i / NS) & 1) ^ 1);
      dec_conv<K, N>(p, sX + xb * C::kXBytes, sB + s * C::kBBytes, sU + s * C::kUBytes, kbase,
                     own_lo, koff, tile * N, wt, cwq);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {                              // per warp: no barrier to strand an aborting warp at
        mbar_arrive(&x_empty[xb]);
        if (kPair) {
          // this warp's rows of both 64-channel blocks of the unit go to the
          // same place in the partner's slot by bulk copy, completing there on
          // b_full; here the arrival expects the partner's matching rows
          constexpr uint32_t kRowBytes = C::SEG * 128;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint32_t off =
                static_cast<uint32_t>(s * C::kBBytes + ((koff >> 6) + kb) * N * 128) + seg_off;
            bulk_copy_to_cluster(sB_peer + off, smem_u32(sB) + off, kRowBytes,
                                 bfull_peer + static_cast<uint32_t>(s * 8));
          }
          mbar_arrive_expect_tx(&b_full[s], 2u * kRowBytes);
        } else {
          mbar_arrive(&b_full[s]);
        }
        mbar_arrive(&job_empty[js]);
      }
    }
    if (kPair) {
      // the last B slots' releases are commits of both CTAs' MMAs arriving here
      // (and they follow the partner's reads of this CTA's copies): let them
      // land before this CTA can exit
      for (int j = i - NS > 0 ? i - NS : 0; j < i; ++j)
        mbar_wait_drain(&b_empty[j % NS], (j / NS) & 1, kDrainNs);
    }
  } else if (warp < 6 + 4 * NE) {
    // ============================ epilogue warpgroups ============================
    const int eg = (warp - 6) >> 2;
    const int qd = warp & 3;
    const int m = qd * 32 + lane;
    const uint32_t t_lane0 = tmem_base + (static_cast<uint32_t>(qd * 32) << 16);
    int cur_unit = -1;
    ChanK kc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    bool fast = true;
    for (int i = eg;; i += NE) {
      const int js = i % kJQ;
      RG_WAIT_OR_ABORT(&job_full[js], (i / kJQ) & 1);
      const int4 job = jobs[js];
      const int unit = job.x, tile = job.y;
      if (unit < 0) break;
      const int c = unit * kM + m;
      const int r0 = tile * N;
      const int nvalid = min(N, p.B - r0);
      const int s = i % NS, ts = i % NT;
      if (unit != cur_unit) {
        cur_unit = unit;
        kc = chan_consts(__bfloat162float(p.b_a[c]), __bfloat162float(p.b_x[c]), p.Lambda[c]);
        fast = __all_sync(0xffffffffu, chan_fast(kc));
      }
      // the previous state of this channel for the job's rows, loaded while the
      // conv and the MMA run (coalesced across lanes)
      float hold[N];
#pragma unroll
      for (int n = 0; n < N; ++n)
        hold[n] = n < nvalid ? p.h[static_cast<size_t>(r0 + n) * p.D + c] : 0.f;
      RG_WAIT_OR_ABORT(&acc_full[ts], (i / NT) & 1);
      tc_fence_after();
      const uint32_t t_lane = t_lane0 + static_cast<uint32_t>(ts * C::kSlotCols);
      const unsigned char *uslot = sU + s * C::kUBytes;
#pragma unroll
      for (int ch = 0; ch < N / 16; ++ch) {
        float za[16], zx[16], uu[16];
        tmem_ld16(t_lane + ch * 16, za);
        tmem_ld16(t_lane + N + ch * 16, zx);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = *reinterpret_cast<const float4 *>(uslot + u_off<N>(m, ch * 4 + q));
          uu[4 * q] = v.x;
          uu[4 * q + 1] = v.y;
          uu[4 * q + 2] = v.z;
          uu[4 * q + 3] = v.w;
        }
        tmem_wait_ld();
        if (ch == N / 16 - 1) {
          // the job's accumulator and u tile are in registers: hand both slots
          // back before the gate math and the global stores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&u_empty[s]);
            mbar_arrive(&tmem_empty[ts]);
          }
        }
#pragma unroll
        for (int pr = 0; pr < 8; ++pr) {
          const int n = ch * 16 + 2 * pr;
          float2 a, beta, la;
          if (fast) {
            gate_pair_fast(make_float2(za[2 * pr], za[2 * pr + 1]),
                           make_float2(zx[2 * pr], zx[2 * pr + 1]),
                           make_float2(uu[2 * pr], uu[2 * pr + 1]), kc, a, beta);
          } else {
            gate_one(za[2 * pr], zx[2 * pr], uu[2 * pr], kc, a.x, beta.x, la.x);
            gate_one(za[2 * pr + 1], zx[2 * pr + 1], uu[2 * pr + 1], kc, a.y, beta.y, la.y);
          }
          const float2 hn = __ffma2_rn(a, make_float2(hold[n], hold[n + 1]), beta);
          if (n < nvalid) {
            const size_t o = static_cast<size_t>(r0 + n) * p.D + c;
            p.h[o] = hn.x;
            p.y_t[o] = __float2bfloat16_rn(hn.x);
          }
          if (n + 1 < nvalid) {
            const size_t o = static_cast<size_t>(r0 + n + 1) * p.D + c;
            p.h[o] = hn.y;
            p.y_t[o] = __float2bfloat16_rn(hn.y);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&job_empty[js]);
    }
  }
#undef RG_WAIT_OR_ABORT

  tc_fence_before();
  // neither CTA of a pair exits while the other may still copy into its
  // shared memory or arrive on its barriers
  if (kPair)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 dec_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

template <int K, int N>
cudaError_t launch_dec_t(const DecArgs &a, cudaStream_t st) {
  using C = DCfg<K, N>;
  auto enc = dec_encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const int bw = a.D / a.H;
  const int R = bw <= 128 ? bw : 256;
  CUtensorMap twa, twx, txt, tring;
  {
    // x_t (B, D): box kXK channels x N rows
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.D), static_cast<cuuint64_t>(a.B)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.D) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::kXK), static_cast<cuuint32_t>(N)};
    cuuint32_t es[2] = {1, 1};
    if (enc(&txt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.x_t), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // ring (B, 3, D): box kXK channels x 1 slot x N rows
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.D), 3, static_cast<cuuint64_t>(a.B)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.D) * 2, static_cast<cuuint64_t>(a.D) * 6};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(C::kXK), 1, static_cast<cuuint32_t>(N)};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tring, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.conv_state, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
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
  DecTcParams p;
  p.x_t = static_cast<const __nv_bfloat16 *>(a.x_t);
  p.conv_w = static_cast<const __nv_bfloat16 *>(a.conv_w);
  p.b_a = static_cast<const __nv_bfloat16 *>(a.b_a);
  p.b_x = static_cast<const __nv_bfloat16 *>(a.b_x);
  p.W_a = static_cast<const __nv_bfloat16 *>(a.W_a);
  p.W_x = static_cast<const __nv_bfloat16 *>(a.W_x);
  p.Lambda = a.Lambda;
  p.ring = static_cast<__nv_bfloat16 *>(a.conv_state);
  p.h = a.h;
  p.y_t = static_cast<__nv_bfloat16 *>(a.y_t);
  p.B = a.B;
  p.D = a.D;
  p.H = a.H;
  p.bw = bw;
  p.pos = a.pos;
  p.n_cg = a.D / kM;
  p.n_tiles = ceil_div(a.B, N);
  p.n_jobs = p.n_cg * p.n_tiles;
  // every CTA is the only reader of its own channels' ring slot (heads up to
  // 128 wide, and CTA pairs), so it rewrites that slot itself
  p.write_ring = 1;
  auto kern = decode_tc_kernel<K, N>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  if (C::kPair) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  // per device, once: the kernel's shared-memory opt-in and how many CTAs (CTA
  // pairs) are resident at once (no attribute call on later steps, which may be
  // captured in a CUDA graph)
  constexpr int kMaxDev = 64;
  static std::atomic<int> slots_of[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int slots = dev < kMaxDev ? slots_of[dev].load(std::memory_order_acquire) : 0;
  if (slots == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    slots = sms;
    if (C::kPair) {
      cfg.gridDim = dim3(2 * (sms / 2));
      if ((e = cudaOccupancyMaxActiveClusters(&slots, kern, &cfg)) != cudaSuccess) return e;
      if (slots < 1) return cudaErrorNotSupported;
    }
    if (dev < kMaxDev) slots_of[dev].store(slots, std::memory_order_release);
  }
  const int items = C::kPair ? p.n_jobs / 2 : p.n_jobs;
  const int groups = items < slots ? items : slots;
  cfg.gridDim = dim3(C::kPair ? 2 * groups : groups);
  return cudaLaunchKernelEx(&cfg, kern, twa, twx, txt, tring, p);
}

}  // namespace

bool tc_decode_supported(int B, int D, int H, int io) { return tc_supported(B, 1, D, H, io); }

int tc_decode_launches(int D, int H) { return D > 0 && H > 0 ? 1 : 0; }

cudaError_t launch_decode_tc(const DecArgs &a, cudaStream_t st) {
  const int bw = a.D / a.H;
  if (bw == 256) return launch_dec_t<256, 16>(a, st);
  return launch_dec_t<128, 16>(a, st);
}

}  // namespace rglru
