// Dense bf16 GEMM on the 5th-generation tensor core (sm_100a) for the recurrent
// block around the layer: C[M x N] = A[M x K] B[K x N], row-major, fp32
// accumulation in TMEM, C stored bf16; optionally C = Y * GeLU(A B) with Y
// (M x N, bf16) read in the epilogue (the block's gating of the layer output
// by GeLU of the gate projection, fused where the gate projection is
// produced; the pages describe the block's gated MLP as GeGeLU-like: "Beyond
// Transformer Architecture: Griffin and Google RecurrentGemma", "Core
// Components of Griffin", 3. Architecture Design).
//
// Two kernels, the same roles: warp 0 issues the TMA copies of A (K-major,
// 128-byte swizzle, boxes of 64 K x 128 rows) and B (MN-major, 128-byte
// swizzle, boxes of 64 columns x 64 K rows) into a ring of stages; warp 1
// issues tcgen05.mma (K = 16 per instruction) into one of two TMEM
// accumulators; two epilogue warpgroups read the accumulator (warp w holds
// TMEM lanes = rows 32 (w mod 4) .. +31, warpgroup g columns 128 g .. +127),
// convert, and store 64 contiguous bytes per row and chunk. Persistent over
// the tiles, K in steps of 64.
//  - gemm_tc2_kernel, when M and N are multiples of 256: clusters of two CTAs
//    share 256 x 256 tiles through the pair MMA (tcgen05 cta_group::2, M =
//    256): each CTA loads 128 rows of A and 128 columns of B per stage, both
//    CTAs' loads complete on the even CTA's barrier, whose MMA thread issues
//    for the pair and commits stage and accumulator releases to both CTAs;
//    each CTA's epilogue stores its 128 rows. Per CTA and stage 32 KB, six
//    stages; a tile's operands cross L2 once per pair, a third less traffic
//    per flop than 128 x 256 tiles on one CTA.
//  - gemm_tc_kernel otherwise: 128 x 256 tiles on one CTA, four stages.
// Every wait is bounded; on expiry the kernel records RGLRU_ERR_TIMEOUT (wait
// site 6) in the status word, drains what it issued and returns.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gelu_as7126.cuh"
#include "kernels.h"
#include "tc_pair.cuh"

namespace rglru {
namespace {

using namespace tc;

#ifndef RGLRU_GEMM_NE
#define RGLRU_GEMM_NE 4
#endif
constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kNE = RGLRU_GEMM_NE;                    // epilogue warpgroups (256 / kNE columns each)
constexpr int kEpiCols = 256 / kNE;
#ifndef RGLRU_GEMM_GELU
#define RGLRU_GEMM_GELU gelu_as7126
#endif
// warps 0 (TMA) and 1 (MMA), the epilogue warpgroups; padded to whole warpgroups
constexpr int kThreads = (64 + kNE * 128 + 127) / 128 * 128;
constexpr int kABytes = kBM * kBK * 2;                // 16 KB
constexpr int kBBytes = kBK * kBN * 2;                // 32 KB (4 blocks of 64 columns)
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kNumBars = 2 * kStages + 4;             // full, empty, acc_full[2], acc_empty[2]
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;
constexpr int kSiteGemm = 6;
static_assert(kSmemBytes <= 232448, "shared memory");

struct GemmParams {
  int M, N, K;
  int n_mt, n_nt, n_tiles;   // CTA pairs: n_tiles work items, the first n_full whole tiles
  int n_full;                // (see pair_item)
  int c_v8, y_v8;            // 1: C (Y) rows may be accessed 32 bytes at a time (N % 16 == 0
                             // and a 32-byte aligned base)
  const __nv_bfloat16 *Y;    // (M, N) or null: C = Y * GeLU(A B)
  __nv_bfloat16 *C;          // (M, N)
  int *dev_status;
};

// 32 bytes at a 32-byte aligned global address (sm_100 256-bit accesses: one
// whole sector per lane).
__device__ __forceinline__ void st_global_v8(void *ptr, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ void ld_global_v8(const void *ptr, uint4 &a, uint4 &b) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z),
                 "=r"(b.w)
               : "l"(ptr));
}

// Y operand of one warp's epilogue: this lane's row, kEpiCols columns from
// c_first, loaded as 8-column vectors before the accumulator is ready (the
// loads then overlap the tile's MMAs instead of the epilogue's arithmetic).
struct EpiY {
  uint4 v[kEpiCols / 8];
};

__device__ __forceinline__ void epilogue_load_y(const GemmParams &p, int row, int c_first,
                                                EpiY &y, int ncols = kEpiCols) {
  if (p.Y == nullptr || row >= p.M) return;
  const __nv_bfloat16 *yr = p.Y + static_cast<size_t>(row) * p.N;
  if (p.y_v8 && c_first % 16 == 0 && c_first + ncols <= p.N) {
    // whole 16-column (32-byte) pieces, 32-byte aligned: one sector per load
#pragma unroll
    for (int q = 0; q < kEpiCols / 8; q += 2)
      if (q * 8 < ncols) ld_global_v8(yr + c_first + q * 8, y.v[q], y.v[q + 1]);
    return;
  }
#pragma unroll
  for (int q = 0; q < kEpiCols / 8; ++q)
    if (q * 8 < ncols && c_first + q * 8 < p.N)
      y.v[q] = *reinterpret_cast<const uint4 *>(yr + c_first + q * 8);
}

// Epilogue of one warp: ncols (a multiple of 32, at most kEpiCols) accumulator
// columns of this lane's row (TMEM address tl: the warp's lane quadrant, the
// first column), converted to bf16 (times Y * GeLU when Y is given, from y) and
// stored from column c_first on, in chunks of 32 columns (64 contiguous bytes
// per row and chunk).
__device__ __forceinline__ void epilogue_rows(const GemmParams &p, uint32_t tl, int row,
                                              int c_first, const EpiY &y, int ncols = kEpiCols) {
#pragma unroll
  for (int ch = 0; ch < kEpiCols / 32; ++ch) {
    if (ch * 32 >= ncols) break;
    const int c0 = c_first + ch * 32;               // first column of this chunk
    float v[32];
    __syncwarp();                                   // tcgen05.ld is warp-collective
    tmem_ld32(tl + static_cast<uint32_t>(ch * 32), v);
    tmem_wait_ld();
    if (row < p.M && c0 < p.N) {
      const size_t off = static_cast<size_t>(row) * p.N + c0;
      const int nq = min(4, (p.N - c0) / 8);       // whole 8-column vectors in range
      if (p.Y != nullptr) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q >= nq) break;
          const uint4 yv = y.v[ch * 4 + q];
          const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float y0 = __uint_as_float(yw[e] << 16);
            const float y1 = __uint_as_float(yw[e] & 0xFFFF0000u);
            v[q * 8 + 2 * e] = y0 * RGLRU_GEMM_GELU(v[q * 8 + 2 * e]);
            v[q * 8 + 2 * e + 1] = y1 * RGLRU_GEMM_GELU(v[q * 8 + 2 * e + 1]);
          }
        }
      }
      if (nq == 4 && p.c_v8) {
        // a whole chunk at a 32-byte aligned address (c0 is a multiple of 32
        // columns): two 256-bit stores, each one whole sector
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat162 h =
                __floats2bfloat162_rn(v[h2 * 16 + 2 * e], v[h2 * 16 + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&h);
          }
          st_global_v8(p.C + off + h2 * 16, w);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q >= nq) break;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h =
                __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&h);
          }
          *reinterpret_cast<uint4 *>(p.C + off + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
               const GemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0 && p.dev_status) atomicCAS(p.dev_status, 0, RGLRU_ERR_UNSUPPORTED);
    return;
  }
  unsigned char *sm = smem_raw;
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + kOffBar);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;
  uint64_t *acc_empty = acc_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
  volatile int *cta_abort = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k_steps = (p.K + kBK - 1) / kBK;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kNE * 4);
    }
    *cta_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto give_up = [&]() {
    if (!*cta_abort) {
      if (p.dev_status) atomicCAS(p.dev_status, 0, RGLRU_ERR_TIMEOUT | (kSiteGemm << 8) |
                                                      (static_cast<int>(blockIdx.x) << 16));
      *cta_abort = 1;
    }
  };

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      int it = 0, last = -1;
      for (int tile = blockIdx.x; tile < p.n_tiles && !*cta_abort; tile += gridDim.x) {
        const int m0 = (tile / p.n_nt) * kBM, n0 = (tile % p.n_nt) * kBN;
        int nb = 0;                                   // B boxes with any column inside N
        while (nb < kBN / 64 && n0 + nb * 64 < p.N) ++nb;
        for (int kb = 0; kb < k_steps; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, cta_abort, kWaitNs)) {
            give_up();
            break;
          }
          unsigned char *st = sm + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kABytes + nb * 64 * kBK * 2));
          tma_load_2d(st, &tmap_a, &full[s], kb * kBK, m0);
          for (int j = 0; j < nb; ++j)
            tma_load_2d(st + kABytes + j * (64 * kBK * 2), &tmap_b, &full[s], n0 + j * 64,
                        kb * kBK);
          last = it;
        }
      }
      if (*cta_abort)
        for (int j = last; j >= 0 && j > last - kStages; --j)
          mbar_wait_drain(&full[j % kStages], (j / kStages) & 1, kDrainNs);
    }
  } else if (warp == 1) {
    // ============================= MMA issuer =============================
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, true);
      int it = 0, lt = 0, last = -1;
      for (int tile = blockIdx.x; tile < p.n_tiles && !*cta_abort; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (!mbar_wait(&acc_empty[buf], ((lt >> 1) & 1) ^ 1, cta_abort, kWaitNs)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kBN);
        bool ok = true;
        for (int kb = 0; kb < k_steps; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], (it / kStages) & 1, cta_abort, kWaitNs)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm + s * kStageBytes);
          // A: K-major rows of 128 B, 8-row groups 1024 B apart; a K step of 16
          // moves 32 B along the row. B: MN-major, 64-column blocks of 64 K rows
          // (8 KB apart), 8-row groups 1024 B apart; a K step moves 16 rows.
          const uint64_t ad = sdesc_sw128(sa, 16, 1024);
          const uint64_t bd = sdesc_sw128(sa + kABytes, 64 * kBK * 2, 1024);
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks)
            mma_bf16(d, ad + static_cast<uint64_t>((ks * 32) >> 4),
                     bd + static_cast<uint64_t>((ks * 16 * 128) >> 4), idesc,
                     (kb > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
          last = it;
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
      }
      if (*cta_abort && last >= 0)
        mbar_wait_drain(&empty[last % kStages], (last / kStages) & 1, kDrainNs);
    }
  } else if (warp < 2 + 4 * kNE) {
    // ============================== epilogue ==============================
    const int g = (warp - 2) >> 2;                  // column group of the tile
    const int qd = warp & 3;                        // TMEM lane quadrant = row block
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const int m0 = (tile / p.n_nt) * kBM, n0 = (tile % p.n_nt) * kBN;
      const int row = m0 + qd * 32 + lane;
      EpiY y;
      epilogue_load_y(p, row, n0 + g * kEpiCols, y);
      if (!mbar_wait(&acc_full[buf], (lt >> 1) & 1, cta_abort, kWaitNs)) {
        give_up();
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                          static_cast<uint32_t>(buf * kBN + g * kEpiCols);
      epilogue_rows(p, tl, row, n0 + g * kEpiCols, y);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ------------------------------------------------------------ CTA pairs ----

constexpr int kPM = 128;                              // rows of A and D per CTA
constexpr int kPN = 128;                              // columns of B per CTA (N = 256 per pair)
constexpr int kPStages = 6;
constexpr int kPABytes = kPM * kBK * 2;               // 16 KB
constexpr int kPBBytes = kBK * kPN * 2;               // 16 KB (2 blocks of 64 columns)
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPOffBar = kPStages * kPStageBytes;
constexpr int kPNumBars = 2 * kPStages + 4;           // full, empty, acc_full[2], acc_empty[2]
constexpr int kPOffMisc = kPOffBar + kPNumBars * 8;
constexpr int kPSmemBytes = kPOffMisc + 64;
static_assert(kPSmemBytes <= 232448, "shared memory");

// Work item w of the pair kernel: whole 256 x 256 tiles first (w < n_full, a
// whole number of waves over the pairs), then each remaining tile as two
// 256 x 128 halves, so that the last wave runs twice as many items of half the
// length. Tiles are numbered with N fastest. Returns the first row, the first
// column and the width (256 or 128).
struct PairItem {
  int m0, n0, nw;
};

__device__ __forceinline__ PairItem pair_item(const GemmParams &p, int w) {
  int f = w, nw = 2 * kPN, half = 0;
  if (w >= p.n_full) {
    f = p.n_full + (w - p.n_full) / 2;
    half = (w - p.n_full) & 1;
    nw = kPN;
  }
  return {(f / p.n_nt) * (2 * kPM), (f % p.n_nt) * (2 * kPN) + half * kPN, nw};
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the alignment is the same in both CTAs, so both return here or neither does
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0 && p.dev_status) atomicCAS(p.dev_status, 0, RGLRU_ERR_UNSUPPORTED);
    return;
  }
  unsigned char *sm = smem_raw;
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + kPOffBar);
  uint64_t *empty = full + kPStages;
  uint64_t *acc_full = empty + kPStages;
  uint64_t *acc_empty = acc_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kPOffMisc);
  volatile int *cta_abort = reinterpret_cast<volatile int *>(sm + kPOffMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();            // 0: issues the pair's MMAs
  const int cid = static_cast<int>(blockIdx.x) >> 1, n_clusters = static_cast<int>(gridDim.x) >> 1;
  const int k_steps = p.K / kBK;
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int *>(cta_abort)), rank ^ 1u);

  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);                         // the even CTA's expect_tx (both CTAs' bytes)
      mbar_init(&empty[s], 1);                        // the pair MMA's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kNE * 4);          // epilogue warps of both CTAs
    }
    *cta_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                                     // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto give_up = [&]() {
    if (!*cta_abort) {
      if (p.dev_status) atomicCAS(p.dev_status, 0, RGLRU_ERR_TIMEOUT | (kSiteGemm << 8) |
                                                      (static_cast<int>(blockIdx.x) << 16));
      *cta_abort = 1;
      st_cluster_u32(peer_abort, 1u);                 // the partner stops at its next wait
    }
  };

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(smem_u32(full), 0u);   // the even CTA's barriers
      int it = 0;
      for (int tile = cid; tile < p.n_tiles && !*cta_abort; tile += n_clusters) {
        const PairItem w = pair_item(p, tile);
        // this CTA's rows of A and its half of the item's columns of B
        const int m0 = w.m0 + static_cast<int>(rank) * kPM;
        const int n0 = w.n0 + static_cast<int>(rank) * (w.nw / 2);
        const int nb = w.nw / 128;                    // 64-column B boxes per CTA
        for (int kb = 0; kb < k_steps; ++kb, ++it) {
          const int s = it % kPStages;
          if (!mbar_wait(&empty[s], ((it / kPStages) & 1) ^ 1, cta_abort, kWaitNs)) {
            give_up();
            break;
          }
          unsigned char *st = sm + s * kPStageBytes;
          if (rank == 0u)
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(2 * (kPABytes + nb * 64 * kBK * 2)));
          const uint32_t fb = full0 + static_cast<uint32_t>(s * 8);
          tma_load_2d_pair(st, &tmap_a, fb, kb * kBK, m0);
          for (int j = 0; j < nb; ++j)
            tma_load_2d_pair(st + kPABytes + j * (64 * kBK * 2), &tmap_b, fb, n0 + j * 64, kb * kBK);
        }
      }
      // the pair MMA's last stage releases arrive here by multicast: let them
      // land before this CTA can exit (bounded)
      for (int j = it - 1; j >= 0 && j >= it - kPStages; --j)
        mbar_wait_drain(&empty[j % kPStages], ((j / kPStages) & 1), kDrainNs);
    }
  } else if (warp == 1) {
    // ============================= MMA issuer =============================
    if (lane == 0 && rank == 0u) {
      constexpr uint32_t idesc_whole = idesc_bf16_f32(2 * kPM, 2 * kPN, false, true);
      constexpr uint32_t idesc_half = idesc_bf16_f32(2 * kPM, kPN, false, true);
      int it = 0, lt = 0;
      for (int tile = cid; tile < p.n_tiles && !*cta_abort; tile += n_clusters, ++lt) {
        const uint32_t idesc = pair_item(p, tile).nw == 2 * kPN ? idesc_whole : idesc_half;
        const int buf = lt & 1;
        if (!mbar_wait(&acc_empty[buf], ((lt >> 1) & 1) ^ 1, cta_abort, kWaitNs)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * 2 * kPN);
        bool ok = true;
        for (int kb = 0; kb < k_steps; ++kb, ++it) {
          const int s = it % kPStages;
          if (!mbar_wait(&full[s], (it / kPStages) & 1, cta_abort, kWaitNs)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm + s * kPStageBytes);
          // A: K-major rows of 128 B, 8-row groups 1024 B apart, a K step of 16
          // moves 32 B along the row; B: MN-major, 64-column blocks of 64 K
          // rows (8 KB apart), a K step moves 16 rows. The same offsets in the
          // odd CTA hold its rows of A and its columns of B.
          const uint64_t ad = sdesc_sw128(sa, 16, 1024);
          const uint64_t bd = sdesc_sw128(sa + kPABytes, 64 * kBK * 2, 1024);
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks)
            mma_bf16_pair(d, ad + static_cast<uint64_t>((ks * 32) >> 4),
                          bd + static_cast<uint64_t>((ks * 16 * 128) >> 4), idesc,
                          (kb > 0 || ks > 0) ? 1u : 0u);
          mma_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[buf], 0x3);
      }
    }
  } else if (warp < 2 + 4 * kNE) {
    // ============================== epilogue ==============================
    const int g = (warp - 2) >> 2;                  // column group of the tile
    const int qd = warp & 3;                        // TMEM lane quadrant = row block
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0u);
    int lt = 0;
    for (int tile = cid; tile < p.n_tiles; tile += n_clusters, ++lt) {
      const int buf = lt & 1;
      const PairItem w = pair_item(p, tile);
      const int row = w.m0 + static_cast<int>(rank) * kPM + qd * 32 + lane;
      const int ncols = w.nw / kNE;                 // this warpgroup's columns of the item
      EpiY y;
      epilogue_load_y(p, row, w.n0 + g * ncols, y, ncols);
      if (!mbar_wait(&acc_full[buf], (lt >> 1) & 1, cta_abort, kWaitNs)) {
        give_up();
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                          static_cast<uint32_t>(buf * 2 * kPN + g * ncols);
      epilogue_rows(p, tl, row, w.n0 + g * ncols, y, ncols);
      tc_fence_before();
      __syncwarp();
      // the accumulator's reads are complete (tcgen05.wait::ld): a relaxed
      // signal to the MMA thread suffices
      if (lane == 0) {
        if (rank == 0u)
          mbar_arrive(&acc_empty[buf]);
        else
          mbar_arrive_cluster_relaxed(acc_empty0 + static_cast<uint32_t>(buf * 8));
      }
    }
  }
  tc_fence_before();
  cluster_sync();                                     // neither CTA exits while the other works
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
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

}  // namespace

bool gemm_tc_supported(int M, int N, int K) {
  // TMA row strides must be multiples of 16 bytes; the epilogue stores 8-column vectors
  return M >= 1 && N >= 8 && K >= 8 && N % 8 == 0 && K % 8 == 0;
}

int launch_gemm_tc(int M, int N, int K, const void *A, const void *B, const void *Y, void *C,
                   int *dev_status, cudaStream_t st) {
  if (!gemm_tc_supported(M, N, K)) return RGLRU_ERR_UNSUPPORTED;
  auto enc = gemm_encode_fn();
  if (enc == nullptr) return RGLRU_ERR_CUDA;
  CUtensorMap ta, tb;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {kBK, kBM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(A), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return RGLRU_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {64, kBK};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(B), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return RGLRU_ERR_CUDA;
  }
  const bool pair = M % (2 * kPM) == 0 && N % (2 * kPN) == 0 && K % kBK == 0;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_mt = pair ? M / (2 * kPM) : ceil_div(M, kBM);
  p.n_nt = pair ? N / (2 * kPN) : ceil_div(N, kBN);
  p.n_tiles = p.n_mt * p.n_nt;
  p.n_full = p.n_tiles;
  p.Y = static_cast<const __nv_bfloat16 *>(Y);
  p.C = static_cast<__nv_bfloat16 *>(C);
  p.c_v8 = (N % 16 == 0 && (reinterpret_cast<uintptr_t>(C) & 31u) == 0) ? 1 : 0;
  p.y_v8 = (Y != nullptr && N % 16 == 0 && (reinterpret_cast<uintptr_t>(Y) & 31u) == 0) ? 1 : 0;
  p.dev_status = dev_status;
  // per device, once: the shared-memory opt-ins, the SM count and how many CTA
  // pairs are resident at once
  constexpr int kMaxDev = 64;
  static std::atomic<int> sms_of[kMaxDev], pairs_of[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
  int sms = dev < kMaxDev ? sms_of[dev].load(std::memory_order_acquire) : 0;
  int pairs = dev < kMaxDev ? pairs_of[dev].load(std::memory_order_acquire) : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (sms == 0) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPSmemBytes) != cudaSuccess)
      return RGLRU_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return RGLRU_ERR_CUDA;
    cfg.gridDim = dim3(2 * (sms / 2));
    if (cudaOccupancyMaxActiveClusters(&pairs, gemm_tc2_kernel, &cfg) != cudaSuccess)
      return RGLRU_ERR_CUDA;
    if (dev < kMaxDev) {
      pairs_of[dev].store(pairs, std::memory_order_release);
      sms_of[dev].store(sms, std::memory_order_release);
    }
  }
  if (pair && pairs > 0) {
    const int clusters = p.n_tiles < pairs ? p.n_tiles : pairs;
    // whole tiles in whole waves; the rest as halves when they then fit one wave
    const int rest = p.n_tiles % clusters;
    p.n_full = p.n_tiles;
    if (rest > 0 && 2 * rest <= clusters) {
      p.n_full = p.n_tiles - rest;
      p.n_tiles = p.n_full + 2 * rest;
    }
    cfg.gridDim = dim3(2 * clusters);
    if (cudaLaunchKernelEx(&cfg, gemm_tc2_kernel, ta, tb, p) != cudaSuccess) return RGLRU_ERR_CUDA;
    return RGLRU_OK;
  }
  if (pair) {                                          // no pair fits: one-CTA tiles
    p.n_mt = ceil_div(M, kBM);
    p.n_nt = ceil_div(N, kBN);
    p.n_tiles = p.n_mt * p.n_nt;
  }
  const int grid = p.n_tiles < sms ? p.n_tiles : sms;
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(ta, tb, p);
  return cudaGetLastError() == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA;
}

}  // namespace rglru
