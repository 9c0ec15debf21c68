// cta_pair.cuh -- device helpers for CTA pairs (clusters of two CTAs on one
// TPC) that share tcgen05 MMAs (`cta_group::2`, sm_100a).
//
// A pair MMA has M = 256: the even CTA of the pair (the leader) issues it for
// both.  A is split by rows (each CTA holds its own 128 rows in shared
// memory), B by columns (each CTA holds half of the N columns), and each CTA
// receives its 128 rows x N of the result in its own TMEM, at the same
// column address.  Both CTAs therefore keep identical shared-memory layouts;
// descriptors built from the leader's addresses address the peer's copy at
// the same offsets.
//
// Synchronisation used by the pair kernels:
//   - tiles: both CTAs load their halves with TMA loads that complete on the
//     leader's barrier (no multicast: each CTA reads its own half);
//   - MMA completion: the leader's commit arrives on the same barrier in
//     both CTAs (commit multicast to the CTA mask 0b11);
//   - consumers of TMEM/shared memory in either CTA arrive on the leader's
//     barriers through the cluster shared window, and the leader waits on
//     them with cluster-scope acquire.
// All waits stay bounded (the same limit and abort flag as bounded_wait).
#pragma once

#include "common.cuh"

namespace fa {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Cluster shared-window address of the same location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}

// All threads of both CTAs (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

// Arrive on a barrier given by its cluster shared-window address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// bounded_wait for a barrier that the other CTA's threads arrive on.
static __device__ __noinline__ bool bounded_wait_cluster_slow(uint32_t bar, uint32_t parity,
                                                              const WaitCtx &w) {
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*w.abort) return false;
      if ((long long)(globaltimer_ns() - t0) > w.limit_ns) {
        *w.abort = 1;
        atomicOr(w.err, kErrTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool bounded_wait_cluster(uint32_t bar, uint32_t parity,
                                                     const WaitCtx &w) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  return bounded_wait_cluster_slow(bar, parity, w);
}

// 3-D tiled load into this CTA's shared memory, completing on `cl_bar`, a
// barrier of either CTA of the pair (cluster shared-window address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void *tmap, uint32_t cl_bar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(cl_bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// TMEM allocation for the pair: the same warp of both CTAs issues these.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

// Pair MMA, kind::f16 (bf16 A and B, f32 accumulate), both operands in
// shared memory; issued by the leader for both CTAs.
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at shared address `bar` of both CTAs when every
// pair MMA issued so far by this thread completes.
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], m;\n\t}" ::"r"(bar)
      : "memory");
}

// The same, arriving on this CTA's barrier only.
__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

}  // namespace fa
