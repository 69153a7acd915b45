// Inline-PTX wrappers for thread-block clusters on sm_100a: the rank of a CTA, peer shared-memory
// addresses, shared-to-peer bulk copies completing on the destination's mbarrier, a tcgen05
// commit that arrives on the same mbarrier in several CTAs, the cluster barrier, and a 2-D TMA
// box load.  Written from the public PTX ISA.  No load here multicasts: every copy has one
// source and one destination.
#pragma once

#include "tc_ptx.cuh"

namespace hys {
namespace tc {

// Rank of this CTA in its cluster.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same shared-memory location in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}

// Bulk copy of `bytes` (a multiple of 16, both ends 16-byte aligned) from this CTA's shared
// memory into another CTA's, completing on an mbarrier in the destination CTA (tx bytes).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, const void* src, uint32_t bytes,
                                                  uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(smem_u32(src)), "r"(bytes), "r"(bar_cluster)
               : "memory");
}

// Arrive on the mbarrier at the same offset in every CTA of `cta_mask` once every tcgen05
// operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit_cluster(uint64_t* bar, uint16_t cta_mask) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"(cta_mask)
               : "memory");
}

// Every thread of every CTA in the cluster arrives, then waits for all of them (the forms
// without .aligned: the threads of a warp need not be converged).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// 2-D tiled load of one box into shared memory, completing on an mbarrier (tx bytes).
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
               : "memory");
}

}  // namespace tc
}  // namespace hys
