// sa_pair2.cuh -- tcgen05 and TMA forms for a pair of CTAs that share one MMA
// (cta_group::2, a 2-CTA thread-block cluster), sm_100a, hand-written inline PTX.
//
// A pair MMA of shape M x N x 16 is issued by the even CTA of the cluster (the leader)
// alone.  Each CTA supplies M/2 rows of A (from its own shared memory or tensor
// memory, at the same address in both) and N/2 rows of B (from its own shared memory,
// same address in both), and receives its M/2 rows of the M x N result in its own
// tensor memory.  The instruction descriptor carries the full M and N.
//
// Every tcgen05 allocation, MMA and commit of one kernel names the same CTA group, so a
// kernel uses either these forms or the single-CTA ones of sa_device.cuh, never both.
// No form here uses TMA multicast.
#pragma once

#include "sa_device.cuh"

namespace sa {

// Issued by one warp of EACH CTA of the pair (the same warp index in both, the same
// shared-memory destination offset): both CTAs receive the same column address.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
// Issued by the allocating warp of each CTA once neither CTA touches the columns again
// (no MMA of the leader in flight, no tcgen05.ld/st of either CTA pending).
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D (+)= A[smem desc] * B[smem desc]^T across the pair, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with A read from each CTA's tensor memory (row m in lane m, K packed two bf16
// per 32-bit column).
__device__ __forceinline__ void umma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// When every pair MMA issued so far by this thread is done, arrive once on the barrier
// at shared-memory offset `bar` in each CTA of the cluster whose bit is set in `cta_mask`
// (bit r = cluster rank r).  A commit, not a copy: no data moves.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

// TMA tile load into THIS CTA's shared memory whose bytes complete on a barrier that
// may live in either CTA of the pair (`bar_cluster`: a shared::cluster address, e.g.
// from mapa_shared(bar, 0) for the leader's).  No multicast: the source is this GPU's
// global memory and the destination is the issuing CTA's own shared memory.
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1, int c2,
                                                 int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

}  // namespace sa
