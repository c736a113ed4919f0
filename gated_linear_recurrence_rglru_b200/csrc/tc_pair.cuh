// sm_100a building blocks for CTA pairs (a cluster of 2 on one GPU), as inline
// PTX: cluster rank and shared::cluster addressing, remote mbarrier arrivals,
// the pair's TMEM allocation, MMA (tcgen05 cta_group::2) and commits, and TMA
// loads that complete on either CTA's barrier (no multicast).
#pragma once

#include "tc_primitives.cuh"

namespace rglru {
namespace tc {

// --------------------------------------------- CTA pairs (cta_group::2) ----
// A cluster of 2 CTAs on one GPU whose tensor cores run one MMA together
// (M = 256: each CTA holds 128 rows of A and of D, and half of B's columns).
// The shared::cluster window addresses the partner's shared memory.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same offset in CTA `rank`'s shared memory.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t caddr, uint32_t x) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(caddr), "r"(x) : "memory");
}

// Arrive on an mbarrier of a CTA of the cluster (shared::cluster address),
// relaxed: a signal that orders nothing, for an arriving thread whose earlier
// accesses the waiter does not depend on (a release at cluster scope would
// first wait for the thread's earlier global stores).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t caddr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}

// Bulk copy (async proxy) of `bytes` from this CTA's shared memory to a CTA of
// the cluster (dst: shared::cluster address); the destination's mbarrier (bar,
// shared::cluster address in that CTA) receives complete_tx of the bytes.
// Addresses 16-byte aligned, bytes a multiple of 16. The source must have been
// written before a fence_proxy_async_smem.
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst, uint32_t src, uint32_t bytes,
                                                     uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// As mma_commit (one CTA's own MMAs, cta_group::1), arriving on the mbarrier at
// `bar`'s offset in every CTA of `cta_mask` (bit r = cluster rank r).
__device__ __forceinline__ void mma_commit_multicast(uint64_t *bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// Every thread of both CTAs arrives (release) and waits (acquire); the
// non-aligned form, so that a warp's threads need not be converged.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// TMEM allocation for a pair: the same warp of both CTAs allocates, both get
// the same columns.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// The pair's MMA, issued by one thread of the even CTA: D (+)= A B^T with the
// descriptors' shared-memory offsets read in both CTAs.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on the mbarrier at `bar`'s offset in every CTA of `cta_mask`
// when the pair's MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// TMA tile load into this CTA's shared memory whose completion (complete_tx)
// goes to an mbarrier of either CTA of the pair (bar: shared::cluster address).
// No multicast: each CTA loads its own tiles.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

}  // namespace tc
}  // namespace rglru
