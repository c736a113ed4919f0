// Fused RG-LRU forward on the 5th-generation tensor core (sm_100a), bf16 I/O.
//
// One pass over HBM: x is read once (TMA), y written once. The layer (its
// definition in include/rglru.h; gates independent of the state, "Beyond
// Transformer Architecture: Griffin and Google RecurrentGemma", "Core
// Components of Griffin", 1. RG-LRU; a memory-bound layer whose kernel should
// optimise HBM accesses, S. De's thread on Griffin) is split into
//   unit = (batch row b, group of 128 output channels), tile = 64 tokens
//   (32 tokens when a head is 256 wide).
// Per tile
//   1. the conv warpgroup computes the width-4 Conv1D token-major (4 channels x
//      4 tokens per step, vector shared-memory rows, packed fp32x2 FMAs) into
//      the K-major bf16 MMA operand and an fp32 copy of the unit's own 128
//      channels of u;
//   2. one thread of another warp issues tcgen05.mma with the gate weights as
//      the A operand (M = 128 output channels) and the conv output as B
//      (N = tokens), so that TMEM lane m holds channel m's two gate
//      pre-activations along time. The weights sit in shared memory for heads
//      up to 128 wide (TMA, 128-byte swizzle, block-diagonal zeros for 64-wide
//      heads) and in TMEM for 256-wide heads, where both gates (128 KB) would
//      leave no shared memory for the pipeline (at each change of unit each gate
//      comes through a 64 KB shared-memory staging buffer by TMA and the conv
//      warpgroup copies it into TMEM);
//   3. an epilogue warpgroup, per lane (channel): sigmoid gates, log-space
//      decay, sqrt(1 - a^2) and a local scan along time from a zero state,
//      keeping the running products P_t = a_1 ... a_t and local states Hl_t
//      in TMEM (pass 1);
//   4. carries the state across tiles with a decoupled look-back over per-tile,
//      per-channel words (prod a, local h) / inclusive state in the workspace —
//      the exact linear scan of S. De's thread ("linear scans instead of
//      parallel scans"), parallel across tiles;
//   5. writes y_t = P_t h_in + Hl_t from the carried state h_in (pass 2, no
//      dependency between tokens).
// Roles: warp 0 claims tiles (per-unit counters in time order; once its own
// unit is done, joining the unit with the most tiles left per CTA claiming it)
// and issues TMA; warp 1 owns TMEM and
// issues the MMAs; warps 2-5 compute the Conv1D of every job; NE epilogue
// warpgroups take the jobs round robin, connected by mbarriers. Tiles
// of a unit are claimed in time order by running CTAs only, so every
// look-back waits on a tile that a running CTA owns. Every wait is bounded:
// on expiry the kernel records RGLRU_ERR_TIMEOUT, raises an abort flag that
// all waits observe, drains what it issued and returns.
#include <cudaTypedefs.h>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_gates.cuh"
#include "tc_primitives.cuh"

namespace rglru {
namespace {

using namespace tc;
using namespace gates;

constexpr int kM = 128;         // output channels per unit (MMA M, TMEM lanes)
constexpr int kJQ = 8;          // job ring depth
constexpr uint64_t kWaitNs = 2000000000ull;   // bound of any wait
// predecessor carry words read per look-back round trip (one L2 latency each)
#ifndef RGLRU_LOOKBACK_WORDS
#define RGLRU_LOOKBACK_WORDS 4
#endif
constexpr int kLB = RGLRU_LOOKBACK_WORDS;
constexpr uint64_t kDrainNs = 200000000ull;   // bound of the drain after an abort

struct TcParams {
  const __nv_bfloat16 *conv_w, *b_a, *b_x;
  const __nv_bfloat16 *W_a, *W_x;            // (H, bw, bw): read directly when A is in TMEM
  const float *Lambda, *h0;
  const __nv_bfloat16 *conv_state_in;
  __nv_bfloat16 *y;
  float *h_T;
  __nv_bfloat16 *conv_state_out;
  int B, T, D, H, bw;
  int n_cg, n_units, n_tiles;
  int *counters, *abort_flag;
  int *workers;                    // per unit: CTAs currently claiming its tiles (a heuristic)
  unsigned long long *carry;       // [unit][tile][128] carry words (see carry_word)
  int *dev_status;
  uint64_t wait_ns;                // bound of every wait
  int fault_tile;                  // testing: tile of unit 0 that never publishes (-1: off)
};

template <int K, int N, int NX, int NE, int NU>
struct Cfg {
  // warps: 0 producer, 1 MMA, 2-5 conv, then NE epilogue warpgroups; the
  // block is padded to whole warpgroups (registers are granted per warpgroup)
  static constexpr int kThreads = (64 + 128 + NE * 128 + 127) / 128 * 128;
  static constexpr int kXRows = N + 3;
  static constexpr int kXBytes = ((kXRows * K * 2) + 1023) / 1024 * 1024;
  // Gate weights (the MMA's A operand, M = 128 output channels x K): in shared
  // memory for K = 128 (TMA, 128-byte swizzle; block-diagonal zeros for 64-wide
  // heads), in TMEM for K = 256, where both gates (128 KB) would not leave
  // shared memory for the pipeline (written by the conv warpgroup)
  static constexpr bool kATmem = (K == 256);
  static constexpr int kABytes = kATmem ? 0 : K * 256;     // one gate: 2 M-blocks x K rows x 128 B
  // staging of one gate's weights (TMA, 128-byte swizzle) on its way into TMEM
  static constexpr int kWBytes = kATmem ? K * 256 : 0;
  static constexpr int kBBytes = N * K * 2;        // K-major conv output, one slot
  // fp32 u of the unit's own channels, channel-major [128][N], for beta
  static constexpr int kUBytes = N * kM * 4;
  static constexpr int kNS = 2;                    // conv -> MMA slots (B operand)
  // conv -> epilogue slots (u tile); with three, the conv of job i waits for
  // pass 1 of job i - 3 rather than of job i - 2
  static constexpr int kNU = NU;
  // TMEM slots: one per epilogue warpgroup and one for the MMA to run ahead
  static constexpr int kNT = NE + 1;
  static constexpr int kOffA = 0;
  static constexpr int kOffW = 2 * kABytes;
  static constexpr int kOffX = kOffW + kWBytes;
  static constexpr int kOffB = kOffX + NX * kXBytes;
  static constexpr int kOffU = kOffB + kNS * kBBytes;
  static constexpr int kOffBar = kOffU + kNU * kUBytes;
  // job_full[JQ], job_empty[JQ], x_full[NX], x_empty[NX], w_full, w_free,
  // b_full[NS], b_empty[NS], u_empty[NU], acc_full[NT], tmem_empty[NT], a_ready, w_mid
  static constexpr int kNumBars = 2 * kJQ + 2 * NX + 2 + 2 * kNS + kNU + 2 * kNT + 2;
  static constexpr int kOffJobs = (kOffBar + kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kOffMisc = kOffJobs + kJQ * 16;
  // the dynamic shared memory base is declared 1024-byte aligned (the kernel
  // checks it), as the 128-byte swizzle of the TMA and MMA tiles needs
  static constexpr int kSmemBytes = kOffMisc + 64;
  static constexpr int kSlotCols = 2 * N;                   // z_a | z_x, then P | Hl
  static constexpr int kACol = kNT * kSlotCols;             // TMEM A: gate a, then gate x
  static constexpr int kUsedCols = kACol + (kATmem ? K : 0);
  static constexpr int kTmemCols = kUsedCols <= 128 ? 128 : (kUsedCols <= 256 ? 256 : 512);
  static_assert((N * (K / 4)) % 128 == 0, "conv mapping");
  static_assert(N % 32 == 0 && K % 128 == 0, "tile shape");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kUsedCols <= 512, "TMEM allocation");
};

// Where a wait gave up, recorded in bits 8-15 of the status word (bits 16-31
// hold the CTA index), so that an expiry names its wait.
enum WaitSite : int {
  kSiteProducer = 1,   // job ring / x slot / weights free (tile claims and TMA)
  kSiteMma = 2,        // job / weights / B operand / TMEM slot (MMA issue)
  kSiteConv = 3,       // job / x tile / B slot / u slot (Conv1D)
  kSiteEpilogue = 4,   // job / accumulator (epilogue)
  kSiteLookBack = 5    // a predecessor tile's carry word
};

__device__ void raise_abort(const TcParams &p, volatile int *cta_abort, int code, int site) {
  if (p.dev_status)
    atomicCAS(p.dev_status, 0, code | (site << 8) | (static_cast<int>(blockIdx.x) << 16));
  atomicExch(p.abort_flag, 1);
  *cta_abort = 1;
}

// Carry word of one (unit, tile, channel), written with one 64-bit store:
//   low 32 bits == 0                -> not published yet (the workspace is zeroed)
//   low 32 bits with the sign bit   -> aggregate: A = prod a over the tile (the
//                                      low bits with the sign cleared), H = local
//                                      state of the tile from zero (high bits)
//   low 32 bits == bits of +1.0f    -> inclusive: the state after the tile (high)
// A is a product of decays in (0, 1], so its sign bit is free; the aggregate
// of a NaN input stays a (NaN) aggregate and never reads as "not published".
constexpr uint32_t kIncTag = 0x3F800000u;
__device__ __forceinline__ unsigned long long carry_agg(float A, float H) {
  return (static_cast<unsigned long long>(__float_as_uint(H)) << 32) |
         (__float_as_uint(A) | 0x80000000u);
}
__device__ __forceinline__ unsigned long long carry_inc(float h) {
  return (static_cast<unsigned long long>(__float_as_uint(h)) << 32) | kIncTag;
}


// Offset (bytes) of (own channel c, 4-token block jb) in the fp32 u tile:
// channel-major rows of N floats whose 16-byte blocks are XOR-permuted by
// (c % 8) ^ (c / 8 % 8). 16-byte accesses are served a quarter warp (8 lanes)
// at a time; the permutation puts any 8 consecutive channels (epilogue
// readers) and any 8 channels 4 apart (conv writers) on distinct banks.
template <int N>
__device__ __forceinline__ uint32_t u_offset(int c, int jb) {
  static_assert(N >= 32, "the permutation needs 8 blocks per row");
  return static_cast<uint32_t>(c * (N * 4) + ((jb ^ ((c & 7) ^ ((c >> 3) & 7))) << 4));
}

// Conv1D of one tile, token-major. Thread t covers the 4 channels
// [4 q, 4 q + 4) of the K range and SEG consecutive tokens; a warp covers 128
// channels of one token segment, so that its shared-memory rows are contiguous
// (no bank conflicts). The loop advances 4 tokens per iteration with a sliding
// window of 4 input rows in registers (a compact loop: the conv shares the
// instruction cache with the epilogue). Writes the bf16 B operand (K-major,
// 128-byte swizzle) and the fp32 u of the unit's own channels
// channel-major into ut (see u_offset). w holds the 4 taps of the 4 channels.
template <int K, int N>
__device__ __forceinline__ void conv_tile(const unsigned char *__restrict__ xs,
                                          unsigned char *__restrict__ bt,
                                          unsigned char *__restrict__ ut, const TcParams &p, int b,
                                          int kbase, int own_lo, int tile, int nvalid,
                                          bool last_tile, int t, const float2 (&w)[4][2]) {
  constexpr int NQ = K / 4;                         // channel quads
  constexpr int SEG = N * NQ / 128;                 // tokens per thread (16)
  static_assert(SEG % 8 == 0, "segments start on a swizzle period");
  const int qd = t % NQ, sg = t / NQ;
  const int kq = qd * 4, nb = sg * SEG;
  const bool own = (kq >= own_lo) && (kq < own_lo + kM);
  const int chq = kbase + kq;                       // first global channel of the quad
  // x tile row r holds token tile * N - 3 + r: the window of output token
  // nb + j is rows nb + j .. nb + j + 3
  // shared-window addresses (32-bit)
  const uint32_t xq = smem_u32(xs) + static_cast<uint32_t>(kq * 2 + nb * K * 2);
  uint2 r0 = lds64(xq);
  uint2 r1 = lds64(xq + K * 2);
  uint2 r2 = lds64(xq + 2 * K * 2);
  if (tile == 0 && nb == 0 && p.conv_state_in != nullptr) {
    const __nv_bfloat16 *cs = p.conv_state_in + static_cast<size_t>(b) * 3 * p.D + chq;
    r0 = __ldg(reinterpret_cast<const uint2 *>(cs));
    r1 = __ldg(reinterpret_cast<const uint2 *>(cs + p.D));
    r2 = __ldg(reinterpret_cast<const uint2 *>(cs + 2 * p.D));
  }
  float2 xw[4][2];
  xw[0][0] = bf2_to_f2(r0.x);
  xw[0][1] = bf2_to_f2(r0.y);
  xw[1][0] = bf2_to_f2(r1.x);
  xw[1][1] = bf2_to_f2(r1.y);
  xw[2][0] = bf2_to_f2(r2.x);
  xw[2][1] = bf2_to_f2(r2.y);
  // B operand: row n = nb + j of the 64-channel block kq / 64; 16-byte chunk
  // (kq % 64) / 8 of the row, XOR-swizzled by n % 8 (= j % 8)
  const uint32_t bq =
      smem_u32(bt) + static_cast<uint32_t>((kq >> 6) * N * 128 + nb * 128 + ((kq & 7) << 1));
  const uint32_t chunk = static_cast<uint32_t>((kq & 63) >> 3);
  // u tile rows of the 4 own channels and their block permutations (x 16 bytes)
  const uint32_t ua = smem_u32(ut);
  uint32_t ubase[4], uperm[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = kq - own_lo + k;
    ubase[k] = ua + static_cast<uint32_t>(c * (N * 4));
    uperm[k] = static_cast<uint32_t>((c & 7) ^ ((c >> 3) & 7)) << 4;
  }
#pragma unroll 1
  for (int jb = 0; jb < SEG; jb += 4) {
    const uint32_t xrow = xq + static_cast<uint32_t>((jb + 3) * K * 2);
    uint2 nr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nr[q] = lds64(xrow + q * K * 2);
    // row nb + jb + q, 16-byte chunk XOR-swizzled by its row % 8; jb % 4 == 0,
    // so (chunk ^ (jb + q)) % 8 == ((chunk ^ jb) % 8) ^ q
    const uint32_t brow = bq + static_cast<uint32_t>(jb * 128);
    const uint32_t cj = ((chunk ^ static_cast<uint32_t>(jb)) & 7u) << 4;
    float uacc[4][4];                               // u of 4 channels x 4 tokens
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xw[(q + 3) & 3][0] = bf2_to_f2(nr[q].x);
      xw[(q + 3) & 3][1] = bf2_to_f2(nr[q].y);
      float2 u[2];
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        float2 acc = __fmul2_rn(w[0][pp], xw[q & 3][pp]);
        acc = __ffma2_rn(w[1][pp], xw[(q + 1) & 3][pp], acc);
        acc = __ffma2_rn(w[2][pp], xw[(q + 2) & 3][pp], acc);
        u[pp] = __ffma2_rn(w[3][pp], xw[(q + 3) & 3][pp], acc);
      }
      sts64(brow + q * 128 + (cj ^ static_cast<uint32_t>(q << 4)), f2_to_bf2(u[0]), f2_to_bf2(u[1]));
      uacc[0][q] = u[0].x;
      uacc[1][q] = u[0].y;
      uacc[2][q] = u[1].x;
      uacc[3][q] = u[1].y;
    }
    if (own) {
      const uint32_t blk = static_cast<uint32_t>((nb + jb) >> 2) << 4;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sts128f(ubase[k] + (blk ^ uperm[k]), uacc[k][0], uacc[k][1], uacc[k][2], uacc[k][3]);
    }
  }
  if (own && last_tile && nb == 0 && p.conv_state_out != nullptr) {
    // the last three inputs x_{T-3}, x_{T-2}, x_{T-1}: rows nvalid .. nvalid + 2
    // (with T < 3 the first of them are conv_state_in rows or zeros: rows 0..2
    // hold them in the tile, or conv_state_in when this is also tile 0)
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const int row = nvalid + r;
      uint2 v = lds64(xq + static_cast<uint32_t>((row - nb) * K * 2));
      if (tile == 0 && row < 3 && p.conv_state_in != nullptr)
        v = __ldg(reinterpret_cast<const uint2 *>(p.conv_state_in +
                                                   (static_cast<size_t>(b) * 3 + row) * p.D + chq));
      *reinterpret_cast<uint2 *>(p.conv_state_out + (static_cast<size_t>(b) * 3 + r) * p.D + chq) = v;
    }
  }
}

// One 16-bit shared-memory load (zero-extended).
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
  return v;
}

// Pass 2 of one tile for one channel (this thread's TMEM lane): y_t =
// P_t h_in + Hl_t for the valid tokens, stored bf16 at a row stride of kD
// channels (a compile-time stride for the common widths, so that the 16
// stores of a chunk take immediate offsets; 0 = runtime D).
template <int N, int kD>
__device__ __forceinline__ void pass2_store(__nv_bfloat16 *yrow, int D, uint32_t t_lane,
                                            int nvalid, float h_in) {
  const size_t ld = kD > 0 ? static_cast<size_t>(kD) : static_cast<size_t>(D);
#pragma unroll 1
  for (int ch = 0; ch < N / 16; ++ch) {
    if (ch * 16 >= nvalid) break;
    float pv[16], hv[16];
    tmem_ld16(t_lane + ch * 16, pv);
    tmem_ld16(t_lane + N + ch * 16, hv);
    tmem_wait_ld();
    __nv_bfloat16 *yc = yrow + static_cast<size_t>(ch * 16) * ld;
    if (ch * 16 + 16 <= nvalid) {
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 v = __ffma2_rn(make_float2(pv[j], pv[j + 1]), f2(h_in),
                                    make_float2(hv[j], hv[j + 1]));
        yc[static_cast<size_t>(j) * ld] = __float2bfloat16_rn(v.x);
        yc[static_cast<size_t>(j + 1) * ld] = __float2bfloat16_rn(v.y);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (ch * 16 + j < nvalid)
          yc[static_cast<size_t>(j) * ld] = __float2bfloat16_rn(fmaf(pv[j], h_in, hv[j]));
    }
  }
}

template <int K, int N, int NX, int NE, int NU>
__global__ void __launch_bounds__(Cfg<K, N, NX, NE, NU>::kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wa,
              const __grid_constant__ CUtensorMap tmap_wx, const TcParams p) {
  using C = Cfg<K, N, NX, NE, NU>;
  constexpr int NS = C::kNS, NT = C::kNT, NUS = C::kNU;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    // the layout relies on the declared alignment; refuse to run without it
    if (threadIdx.x == 0 && p.dev_status) atomicCAS(p.dev_status, 0, RGLRU_ERR_UNSUPPORTED);
    return;
  }
  unsigned char *sm = smem_raw;
  unsigned char *sA = sm + C::kOffA;
  unsigned char *sW = sm + C::kOffW;
  unsigned char *sX = sm + C::kOffX;
  unsigned char *sB = sm + C::kOffB;
  unsigned char *sU = sm + C::kOffU;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
  uint64_t *job_full = bars;
  uint64_t *job_empty = job_full + kJQ;
  uint64_t *x_full = job_empty + kJQ;
  uint64_t *x_empty = x_full + NX;
  uint64_t *w_full = x_empty + NX;
  uint64_t *w_free = w_full + 1;                    // MMAs reading the old weights are done
  uint64_t *b_full = w_free + 1;                    // [NS] conv -> MMA
  uint64_t *b_empty = b_full + NS;                  // [NS] MMA -> conv
  uint64_t *u_empty = b_empty + NS;                 // [NU] epilogue pass 1 -> conv
  uint64_t *acc_full = u_empty + NUS;               // [NT] MMA -> epilogue
  uint64_t *tmem_empty = acc_full + NT;             // [NT] epilogue pass 2 -> MMA
  uint64_t *a_ready = tmem_empty + NT;              // conv warpgroup wrote TMEM weights -> MMA
  uint64_t *w_mid = a_ready + 1;                    // staged gate a read (TMEM weights)
  int4 *jobs = reinterpret_cast<int4 *>(sm + C::kOffJobs);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::kOffMisc);
  volatile int *cta_abort = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 4);
  volatile int *bcast = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 8);  // [NE][2]
  // phases of w_full armed so far (producer and conv warpgroup): an aborting CTA
  // waits for the last one before it exits, so that no weight copy is in flight
  int *w_armed = reinterpret_cast<int *>(sm + C::kOffMisc + 48);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- set-up: barriers, zero weight tiles (block-diagonal zeros), TMEM ----
  if (tid == 0) {
    for (int i = 0; i < kJQ; ++i) {
      mbar_init(&job_full[i], 1);
      mbar_init(&job_empty[i], 9);                  // 4 conv warps, MMA, 4 epilogue warps
    }
    for (int i = 0; i < NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 4);                    // 4 conv warps, or 4 epilogue warps
    }
    mbar_init(w_full, 1);
    // shared-memory weights: the MMA thread; TMEM weights: the conv warps' copy
    mbar_init(w_free, C::kATmem ? 4 : 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&b_full[i], 4);                     // 4 conv warps
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < NUS; ++i) mbar_init(&u_empty[i], 4);   // 4 epilogue warps
    for (int i = 0; i < NT; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&tmem_empty[i], 4);                 // 4 epilogue warps
    }
    mbar_init(a_ready, 4);                          // 4 conv warps
    mbar_init(w_mid, 4);                            // 4 conv warps
    *cta_abort = 0;
    *w_armed = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_wa);
    prefetch_tmap(&tmap_wx);
  }
  {
    uint4 *a4 = reinterpret_cast<uint4 *>(sA);
    for (int i = tid; i < 2 * C::kABytes / 16; i += C::kThreads) a4[i] = make_uint4(0, 0, 0, 0);
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

#define RG_WAIT_OR_ABORT(bar, par)                                          \
  if (!mbar_wait((bar), (par), cta_abort, p.wait_ns)) {                       \
    if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT, wait_site); \
    break;                                                                  \
  }

  if (warp == 0) {
    // =============================== producer ===============================
    constexpr int wait_site = kSiteProducer;
    // The whole warp runs this loop (all decisions are warp-uniform): all
    // lanes wait on the ring barriers, lane 0 takes the counter, all lanes
    // scan the other units in parallel once the current unit is done, and
    // lane 0 alone writes the job, arrives and issues the copies. A tile is
    // claimed only once its x slot is free, so that tiles are claimed close
    // to the time they are processed and a look-back rarely waits on a tile
    // that sits claimed in another CTA's queue.
    {
      int unit = blockIdx.x % p.n_units, w_unit = -1;
      int i = 0, last_x_job = -1;
      if (lane == 0) atomicAdd(&p.workers[unit], 1);
      uint32_t wfree_phase = 0;
      for (;; ++i) {
        const int js = i % kJQ, xb = i % NX;
        RG_WAIT_OR_ABORT(&job_empty[js], ((i / kJQ) & 1) ^ 1);
        RG_WAIT_OR_ABORT(&x_empty[xb], ((i / NX) & 1) ^ 1);
        int tile = -1;
        while (unit >= 0) {
          int t = 0;
          if (lane == 0) t = atomicAdd(&p.counters[unit], 1);
          t = __shfl_sync(0xffffffffu, t, 0);
          if (t < p.n_tiles) {
            tile = t;
            break;
          }
          // this unit is done: join the unit that would finish last, the one
          // with the most tiles left per CTA claiming it (with this one), so
          // that units end together and CTAs change unit (a TMEM weight reload
          // and a pipeline drain for 256-wide heads) as rarely as possible;
          // ties broken by distance from a per-CTA starting point. Counters and
          // worker counts are read from L2 without ordering: a stale value only
          // makes a worse choice, the claim itself is the atomic.
          if (lane == 0) atomicSub(&p.workers[unit], 1);
          const int rot = static_cast<int>((blockIdx.x * 37u) % static_cast<unsigned>(p.n_units));
          unsigned key = 0;                       // (16 x tiles left per CTA << 16) | (65535 - distance)
          for (int u0 = 0; u0 < p.n_units; u0 += 128) {
            int l[4], wk[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int u = u0 + q * 32 + lane;
              l[q] = u < p.n_units ? p.n_tiles - __ldcg(p.counters + u) : 0;
              wk[q] = u < p.n_units ? __ldcg(p.workers + u) : 0;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int u = u0 + q * 32 + lane;
              if (l[q] > 0) {
                const int dist = u >= rot ? u - rot : u + p.n_units - rot;
                const int per = min(l[q] * 16 / (max(wk[q], 0) + 1), 65535);
                const unsigned k = (static_cast<unsigned>(per) << 16) |
                                   static_cast<unsigned>(65535 - min(dist, 65535));
                key = max(key, k);
              }
            }
          }
          key = __reduce_max_sync(0xffffffffu, key);
          if (key == 0) {
            unit = -1;
          } else {
            const int dist = 65535 - static_cast<int>(key & 0xFFFFu);
            unit = rot + dist < p.n_units ? rot + dist : rot + dist - p.n_units;
            if (lane == 0) atomicAdd(&p.workers[unit], 1);
          }
        }
        unit = __shfl_sync(0xffffffffu, *cta_abort ? -1 : unit, 0);
        const int reload = (unit >= 0 && unit != w_unit) ? 1 : 0;
        if (lane == 0) {
          jobs[js] = make_int4(unit, tile, reload, 0);
          mbar_arrive(&job_full[js]);
        }
        if (unit < 0) {
          // one terminal job per epilogue warpgroup that may still wait for a job
          for (int e = 1; e < NE; ++e) {
            const int je = i + e;
            if (!mbar_wait(&job_empty[je % kJQ], ((je / kJQ) & 1) ^ 1, cta_abort, p.wait_ns)) break;
            if (lane == 0) {
              jobs[je % kJQ] = make_int4(-1, -1, 0, 0);
              mbar_arrive(&job_full[je % kJQ]);
            }
          }
          break;
        }
        const int b = unit / p.n_cg, cg = unit % p.n_cg;
        if (reload && !C::kATmem) {
          if (i > 0) {
            // the MMA warp signals once the MMAs of job i-1 (the last readers of
            // the weights in shared memory) have completed
            RG_WAIT_OR_ABORT(w_free, wfree_phase);
            wfree_phase ^= 1;
          }
          if (lane == 0) {
            atomicAdd(w_armed, 1);
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
          }
        }
        if (reload && C::kATmem) {
          // gate a of the new unit into the staging buffer, ahead of its job; the
          // conv warpgroup copies it into TMEM, then stages gate x itself
          if (i > 0) {
            RG_WAIT_OR_ABORT(w_free, wfree_phase);  // the previous unit's staging is copied
            wfree_phase ^= 1;
          }
          if (lane == 0) {
            atomicAdd(w_armed, 1);
            mbar_arrive_expect_tx(w_full, static_cast<uint32_t>(C::kWBytes));
            for (int ma = 0; ma < 2; ++ma)
              tma_load_2d(sW + ma * (K * 128), &tmap_wa, w_full, (cg & 1) * 128 + 64 * ma,
                          (cg >> 1) * 256);
          }
        }
        if (reload) w_unit = unit;
        const int kbase = p.bw <= 128 ? cg * kM : (cg >> 1) * 256;
        if (lane == 0) {
          mbar_arrive_expect_tx(&x_full[xb], static_cast<uint32_t>(C::kXRows * K * 2));
          tma_load_3d(sX + xb * C::kXBytes, &tmap_x, &x_full[xb], kbase, tile * N - 3, b);
        }
        last_x_job = i;
      }
      if (lane == 0 && *cta_abort) {
        // drain: let every TMA this thread issued land before the CTA exits
        for (int j = last_x_job; j >= 0 && j > last_x_job - NX; --j)
          mbar_wait_drain(&x_full[j % NX], (j / NX) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    constexpr int wait_site = kSiteMma;
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
              // MMAs complete in order: job i-1 done => every read of the old weights done
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
        mma_commit(&b_empty[s]);
        last_commit = i;
        mbar_arrive(&job_empty[js]);
      }
      if (*cta_abort && last_commit >= 0)
        mbar_wait_drain(&acc_full[last_commit % NT], (last_commit / NT) & 1, kDrainNs);
    }
  } else if (warp < 6) {
    // ============================ conv warpgroup ============================
    constexpr int wait_site = kSiteConv;
    const int wt = tid - 64;                      // 0 .. 127
    int cur_unit = -1;
    uint32_t wfull_phase = 0, wmid_phase = 0;     // staged-weight barriers (TMEM weights)
    float2 cwq[4][2];                             // conv taps of this thread's channel quad
    for (int i = 0;; ++i) {
      const int js = i % kJQ;
      RG_WAIT_OR_ABORT(&job_full[js], (i / kJQ) & 1);
      const int4 job = jobs[js];
      const int unit = job.x, tile = job.y;
      if (unit < 0) break;
      const int b = unit / p.n_cg, cg = unit % p.n_cg;
      const int kbase = p.bw <= 128 ? cg * kM : (cg >> 1) * 256;
      const int own_lo = p.bw <= 128 ? 0 : (cg & 1) * kM;
      const int nvalid = min(N, p.T - tile * N);
      if (unit != cur_unit) {
        cur_unit = unit;
        const int chq = kbase + (wt % (K / 4)) * 4;
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
          const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.conv_w + tap * p.D + chq));
          cwq[tap][0] = bf2_to_f2(raw.x);
          cwq[tap][1] = bf2_to_f2(raw.y);
        }
        if (C::kATmem) {
          // This unit's gate weights into TMEM (the A operand): lane m (output
          // channel cg*128 + m) holds W[h][k][j] for k = 0..K-1, two per column.
          // Each gate comes through the staging buffer (TMA, 128-byte swizzle,
          // MN-major: per 64-channel block ma, row k of 128 B, 16-byte chunk
          // (m % 64) / 8 stored at chunk ^ (k % 8); a warp's 32 channels read 64
          // bytes of one row: no bank conflicts): gate a was staged by the tile
          // claimer ahead of this job, gate x is staged here once every warp has
          // copied gate a. Every MMA of earlier jobs has read the old weights once
          // the accumulator of job i-1 is complete (MMAs complete in issue order).
          RG_WAIT_OR_ABORT(w_full, wfull_phase);        // gate a staged
          wfull_phase ^= 1;
          if (i > 0) RG_WAIT_OR_ABORT(&acc_full[(i - 1) % NT], ((i - 1) / NT) & 1);
          const int qd = warp & 3;                  // this warp's TMEM lane quadrant
          const int m = qd * 32 + lane;             // output channel within the unit
          const uint32_t tq = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                              static_cast<uint32_t>(C::kACol);
          const uint32_t wsrc = smem_u32(sW) +
                                static_cast<uint32_t>((m >> 6) * (K * 128) + ((m & 7) << 1));
          const uint32_t mchunk = static_cast<uint32_t>((m & 63) >> 3);
          bool ok = true;
#pragma unroll 1
          for (int g = 0; g < 2 && ok; ++g) {
            if (g == 1) {
              // every warp has read gate a: one thread stages gate x
              __syncwarp();
              if (lane == 0) mbar_arrive(w_mid);
              if (warp == 2 && lane == 0) {
                if (mbar_wait(w_mid, wmid_phase, cta_abort, p.wait_ns)) {
                  atomicAdd(w_armed, 1);
                  mbar_arrive_expect_tx(w_full, static_cast<uint32_t>(C::kWBytes));
                  for (int ma = 0; ma < 2; ++ma)
                    tma_load_2d(sW + ma * (K * 128), &tmap_wx, w_full, (cg & 1) * 128 + 64 * ma,
                                (cg >> 1) * 256);
                } else if (!*cta_abort) {
                  raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT, wait_site);
                }
              }
              __syncwarp();                         // warp 2's lane 0 rejoins its warp
              wmid_phase ^= 1;
              ok = mbar_wait(w_full, wfull_phase, cta_abort, p.wait_ns);   // gate x staged
              wfull_phase ^= 1;
              if (!ok) break;
            }
            __syncwarp();                           // tcgen05.st is warp-collective
#pragma unroll 1
            for (int cc = 0; cc < K / 64; ++cc) {
              uint32_t v[32];
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                const uint32_t k = static_cast<uint32_t>(cc * 64 + 2 * q);   // even: k % 8 = 2q % 8
                const uint32_t lo = lds_u16(wsrc + k * 128 + ((mchunk ^ (k & 7)) << 4));
                const uint32_t hi = lds_u16(wsrc + (k + 1) * 128 + ((mchunk ^ ((k + 1) & 7)) << 4));
                v[q] = lo | (hi << 16);
              }
              tmem_st32u(tq + static_cast<uint32_t>(g * (K / 2) + cc * 32), v);
            }
          }
          if (!ok) {
            if (!*cta_abort) raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT, wait_site);
            break;
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(a_ready);
            mbar_arrive(w_free);                    // the staging buffer may be reloaded
          }
        }
      }
      const int s = i % NS, xb = i % NX, us = i % NUS;
      RG_WAIT_OR_ABORT(&x_full[xb], (i / NX) & 1);
      RG_WAIT_OR_ABORT(&b_empty[s], ((i / NS) & 1) ^ 1);
      RG_WAIT_OR_ABORT(&u_empty[us], ((i / NUS) & 1) ^ 1);
      conv_tile<K, N>(sX + xb * C::kXBytes, sB + s * C::kBBytes, sU + us * C::kUBytes,
                                 p, b, kbase, own_lo, tile, nvalid, tile == p.n_tiles - 1, wt,
                                 cwq);
      // each warp hands its part over on its own: no barrier that an aborting
      // warp could leave the others waiting at
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&x_empty[xb]);
        mbar_arrive(&b_full[s]);
        mbar_arrive(&job_empty[js]);
      }
    }
  } else if (warp < 6 + 4 * NE) {
    // ========================== epilogue warpgroups ==========================
    constexpr int wait_site = kSiteEpilogue;
    // Epilogue warpgroup e takes jobs e, e + NE, ...; each of its 4 warps owns
    // one TMEM quadrant (32 channels, one per lane) and works on its own: per
    // job, pass 1, the publication of each channel's aggregate, the carry
    // (look-back over its channels' words) and pass 2. Three warpgroups keep
    // three jobs in flight while the MMA fills the fourth TMEM slot.
    const int eg = (warp - 6) >> 2;               // 0 .. NE-1
    const int qd = warp & 3;                      // TMEM quadrant
    const int m = qd * 32 + lane;                 // TMEM lane == output channel in unit
    const uint32_t t_lane0 = tmem_base + (static_cast<uint32_t>(qd * 32) << 16);
    int cur_unit = -1;
    ChanK kc{};
    bool fast = true;

    for (int i = eg;; i += NE) {
      const int js = i % kJQ;
      RG_WAIT_OR_ABORT(&job_full[js], (i / kJQ) & 1);
      const int4 job = jobs[js];
      const int unit = job.x, tile = job.y;
      if (unit < 0) break;
      const int b = unit / p.n_cg, cg = unit % p.n_cg;
      const int c = cg * kM + m;                  // own output channel
      const int nvalid = min(N, p.T - tile * N);
      const int us = i % NUS, ts = i % NT;
      const uint32_t t_lane = t_lane0 + static_cast<uint32_t>(ts * C::kSlotCols);
      if (unit != cur_unit) {
        cur_unit = unit;
        kc = chan_consts(__bfloat162float(p.b_a[c]), __bfloat162float(p.b_x[c]), p.Lambda[c]);
        fast = __all_sync(0xffffffffu, chan_fast(kc));
      }
      RG_WAIT_OR_ABORT(&acc_full[ts], (i / NT) & 1);
      tc_fence_after();
      // own channel's u: the fp32 tile from the conv warpgroup; this channel's
      // row of it and its block permutation (x 16 bytes)
      const uint32_t urow = smem_u32(sU + us * C::kUBytes) + static_cast<uint32_t>(m * (N * 4));
      const uint32_t uperm = static_cast<uint32_t>((m & 7) ^ ((m >> 3) & 7)) << 4;
      // ---- pass 1: gates, decay, local scan from zero; (P_t, Hl_t) -> TMEM ----
      // 16 tokens per TMEM round trip, the gate math two tokens at a time in
      // fp32x2 instructions. Tokens past the end of the sequence (last tile)
      // are computed like the others (their x rows read as zeros) and never
      // used: the tile's aggregate is read back at the last valid token.
      float Hl = 0.f, P = 1.f;
#pragma unroll 1
      for (int ch = 0; ch < N / 16; ++ch) {
        float za[16], zx[16], uu[16];
        tmem_ld16(t_lane + ch * 16, za);
        tmem_ld16(t_lane + N + ch * 16, zx);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = lds128f(urow + (static_cast<uint32_t>((ch * 4 + q) << 4) ^ uperm));
          uu[4 * q] = v.x; uu[4 * q + 1] = v.y; uu[4 * q + 2] = v.z; uu[4 * q + 3] = v.w;
        }
        if (ch == N / 16 - 1) {
          // the last reads of the u tile are issued: hand the slot back
          __syncwarp();
          if (lane == 0) mbar_arrive(&u_empty[us]);
        }
        tmem_wait_ld();
        if (fast) {
#pragma unroll
          for (int pr = 0; pr < 8; ++pr) {
            float2 a, beta;
            gate_pair_fast(make_float2(za[2 * pr], za[2 * pr + 1]),
                           make_float2(zx[2 * pr], zx[2 * pr + 1]),
                           make_float2(uu[2 * pr], uu[2 * pr + 1]), kc, a, beta);
            Hl = fmaf(a.x, Hl, beta.x);
            P *= a.x;
            za[2 * pr] = P;
            zx[2 * pr] = Hl;
            Hl = fmaf(a.y, Hl, beta.y);
            P *= a.y;
            za[2 * pr + 1] = P;
            zx[2 * pr + 1] = Hl;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float a, beta, la;
            gate_one(za[j], zx[j], uu[j], kc, a, beta, la);
            Hl = fmaf(a, Hl, beta);
            P *= a;
            za[j] = P;
            zx[j] = Hl;
          }
        }
        tmem_st16(t_lane + ch * 16, za);
        tmem_st16(t_lane + N + ch * 16, zx);
      }
      tmem_wait_st();
      // the tile's aggregate over its valid tokens: (prod a, local state)
      float A = P, Hag = Hl;
      if (nvalid < N) {
        A = tmem_ld1(t_lane + (nvalid - 1));
        Hag = tmem_ld1(t_lane + N + (nvalid - 1));
        tmem_wait_ld();
      }
      // publish this channel's word: inclusive for the first tile of a
      // sequence (h0 is known), else the aggregate
      {
        const size_t wix = (static_cast<size_t>(unit) * p.n_tiles + tile) * kM + m;
        const bool silent = (unit == 0 && tile == p.fault_tile);
        if (!silent) {
          if (tile == 0) {
            const float h0v = p.h0 != nullptr ? p.h0[static_cast<size_t>(b) * p.D + c] : 0.f;
            st_relaxed_u64(p.carry + wix, carry_inc(fmaf(A, h0v, Hag)));
          } else {
            st_relaxed_u64(p.carry + wix, carry_agg(A, Hag));
          }
        }
      }
      // ---- carry: the state entering this tile ----
      unsigned long long *cw = p.carry + static_cast<size_t>(unit) * p.n_tiles * kM + m;
      float h_in = 0.f;
      if (tile == 0) {
        if (p.h0 != nullptr) h_in = p.h0[static_cast<size_t>(b) * p.D + c];
      } else {
        // Look back along this lane's channel, kLB words per round trip: fold
        // aggregates until an inclusive word; an unpublished word ends the
        // round and is read again in the next.
        float mult = 1.f, add = 0.f;
        int k = tile - 1;                         // next tile to read
        bool done = false;
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
          if (!done) {
            unsigned long long w[kLB];
#pragma unroll
            for (int q = 0; q < kLB; ++q)
              w[q] = (k - q >= 0) ? ld_relaxed_u64(cw + static_cast<size_t>(k - q) * kM) : 0ull;
            bool stop = false;
#pragma unroll
            for (int q = 0; q < kLB; ++q) {
              if (stop) continue;
              const uint32_t lo = static_cast<uint32_t>(w[q]);
              const float hi = __uint_as_float(static_cast<uint32_t>(w[q] >> 32));
              if (lo == 0u) {
                stop = true;                      // not yet published: read tile k again
              } else if (lo & 0x80000000u) {
                add = fmaf(mult, hi, add);        // aggregate
                mult *= __uint_as_float(lo & 0x7FFFFFFFu);
                --k;
              } else {
                h_in = fmaf(mult, hi, add);       // inclusive
                done = true;
                stop = true;
              }
            }
          }
          if (__all_sync(0xffffffffu, done)) break;
          const bool give_up = *cta_abort || *(volatile const int *)p.abort_flag ||
                               (globaltimer_ns() - t0 > p.wait_ns);
          if (__any_sync(0xffffffffu, give_up)) {
            if (lane == 0 && !*cta_abort)
              raise_abort(p, cta_abort, RGLRU_ERR_TIMEOUT, kSiteLookBack);
            *cta_abort = 1;
            h_in = 0.f;
            break;
          }
          // no sleep between rounds: each round is one L2 round trip already, and
          // a sleep only delays seeing the predecessor's word (measured: 16 to
          // 256 ns sleeps were 1 to 2 % slower on long sequences)
        }
        if (!(unit == 0 && tile == p.fault_tile))
          st_relaxed_u64(cw + static_cast<size_t>(tile) * kM, carry_inc(fmaf(A, h_in, Hag)));
      }
      // ---- pass 2: y_t = P_t h_in + Hl_t ----
      __nv_bfloat16 *yrow = p.y + (static_cast<size_t>(b) * p.T + tile * N) * p.D + c;
      switch (p.D) {
        case 1024: pass2_store<N, 1024>(yrow, p.D, t_lane, nvalid, h_in); break;
        case 2560: pass2_store<N, 2560>(yrow, p.D, t_lane, nvalid, h_in); break;
        case 4096: pass2_store<N, 4096>(yrow, p.D, t_lane, nvalid, h_in); break;
        default: pass2_store<N, 0>(yrow, p.D, t_lane, nvalid, h_in); break;
      }
      if (tile == p.n_tiles - 1 && p.h_T != nullptr)
        p.h_T[static_cast<size_t>(b) * p.D + c] = fmaf(A, h_in, Hag);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tmem_empty[ts]);
        mbar_arrive(&job_empty[js]);
      }
    }
  }
#undef RG_WAIT_OR_ABORT

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && *cta_abort && *w_armed > 0)
    mbar_wait_drain(w_full, static_cast<uint32_t>(*w_armed - 1) & 1u, kDrainNs);
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
  size_t off_counters, off_workers, off_abort, off_carry, total;
};

TcLayout tc_layout(int B, int T, int D, int H) {
  TcLayout L{};
  const int bw = D / H;
  L.n_cg = D / kM;
  L.n_units = B * L.n_cg;
  L.n_tiles = ceil_div(T, tile_tokens(bw));
  L.off_counters = 0;
  L.off_workers = static_cast<size_t>(L.n_units) * 4;
  L.off_abort = L.off_workers + static_cast<size_t>(L.n_units) * 4;
  L.off_carry = align_up(L.off_abort + 4, 256);
  // one 8-byte carry word per (unit, tile, channel); all of it starts at zero
  L.total = align_up(L.off_carry + static_cast<size_t>(L.n_units) * L.n_tiles * kM * 8, 256);
  return L;
}

template <int K, int N, int NX, int NE, int NU>
cudaError_t launch_tc_t(const FwdArgs &a, const TcLayout &L, void *ws, cudaStream_t st) {
  using C = Cfg<K, N, NX, NE, NU>;
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
  p.W_a = static_cast<const __nv_bfloat16 *>(a.W_a);
  p.W_x = static_cast<const __nv_bfloat16 *>(a.W_x);
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
  p.workers = reinterpret_cast<int *>(w + L.off_workers);
  p.carry = reinterpret_cast<unsigned long long *>(w + L.off_carry);
  p.dev_status = a.dev_status;
  p.wait_ns = a.wait_ns ? a.wait_ns : kWaitNs;
  p.fault_tile = a.fault_tile;

  cudaError_t e = cudaMemsetAsync(ws, 0, L.total, st);
  if (e != cudaSuccess) return e;
  auto kern = fwd_tc_kernel<K, N, NX, NE, NU>;
  // per device, once: the kernel's shared-memory opt-in and the SM count
  constexpr int kMaxDev = 64;
  static std::atomic<int> sms_of[kMaxDev];
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  int sms = dev < kMaxDev ? sms_of[dev].load(std::memory_order_acquire) : 0;
  if (sms == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    if (dev < kMaxDev) sms_of[dev].store(sms, std::memory_order_release);
  }
  const long jobs = static_cast<long>(L.n_units) * L.n_tiles;
  const int grid = static_cast<int>(jobs < sms ? jobs : sms);
  if (a.ev_begin != nullptr && (e = cudaEventRecord(a.ev_begin, st)) != cudaSuccess) return e;
  kern<<<grid, C::kThreads, C::kSmemBytes, st>>>(tx, twa, twx, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.ev_end != nullptr) return cudaEventRecord(a.ev_end, st);
  return cudaSuccess;
}

}  // namespace

bool tc_supported(int B, int T, int D, int H, int io) {
  if (io != RGLRU_IO_BF16) return false;
  if (D % kM != 0 || D % H != 0) return false;
  // the unit index of a steal decision is carried in 16 bits
  if (static_cast<long long>(B) * (D / kM) > 65535) return false;
  const int bw = D / H;
  return bw == 64 || bw == 128 || bw == 256;
}

size_t tc_workspace_bytes(int B, int T, int D, int H) { return tc_layout(B, T, D, H).total; }

cudaError_t launch_fwd_tc(const FwdArgs &a, void *ws, cudaStream_t st) {
  const int bw = a.D / a.H;
  const TcLayout L = tc_layout(a.B, a.T, a.D, a.H);
  if (bw == 256) return launch_tc_t<256, 32, 3, 3, 3>(a, L, ws, st);
  return launch_tc_t<128, 64, 2, 3, 3>(a, L, ws, st);
}

}  // namespace rglru
