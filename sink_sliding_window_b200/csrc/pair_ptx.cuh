// PTX wrappers for kernels launched as clusters of two CTAs whose tcgen05
// MMAs run on the CTA pair (.cta_group::2): one MMA of M = 256 rows takes A
// as 128 rows from each CTA (shared memory or TMEM), B as N/2 columns from
// each CTA's shared memory, and writes each CTA's 128 rows x N into that
// CTA's TMEM.  Every tcgen05 instruction of a kernel that uses these carries
// .cta_group::2 (allocation, MMA, commit); the .cta_group::1 forms in ptx.cuh
// are for the other kernels.
#pragma once
#include "ptx.cuh"

namespace sa {

// Rank of this CTA in its cluster (0 or 1 for a pair).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the object at shared::cta address `a` in the
// cluster's CTA of rank `rank` (a shared::cta address of the executing CTA
// is itself a valid shared::cluster address of that CTA).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}

// Every thread of both CTAs: this CTA's earlier shared-memory writes (barrier
// initialisation included) become visible to the peer, and no thread goes on
// before all threads of the cluster arrived.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or
// the peer's), releasing this thread's earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// Parity wait on a barrier of this CTA with cluster-scope acquire, for
// barriers whose arrivals come from the peer CTA (its threads, its TMA loads,
// or commits of MMAs the peer issued).  Same suspend hint as ptx.cuh.
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait with the same contract as mbar_wait (ptx.cuh): gives up after
// kWaitLimitNs or when this CTA's abort flag is raised, recording `code`.
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                             int code) {
  if (mbar_try_wait_cl(bar, parity, 0)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_cl(bar, parity, kWaitSleepNs)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicCAS(err, 0, code);
      *abort = 1;
      return false;
    }
  }
}

// 3-D tiled TMA load into this CTA's shared memory whose completion (the
// box's bytes) is signalled on a barrier of either CTA of the pair, given by
// its shared::cluster address.  Each CTA loads its own boxes; no load is
// shared between the CTAs.
// x keeps the 16-byte alignment TMA needs (callers pass 0 or 32 bf16).
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// TMEM allocation for a CTA pair: one warp of each CTA (the same warp index)
// issues it with the same destination offset; both CTAs get the same columns.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Arrives once on the barrier at shared::cluster address `bar_cluster` (this
// CTA's or the peer's) when every pair MMA this thread issued so far is done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Pair MMA, A and B from shared memory (kind::f16, fp32 accumulate).
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair MMA, A from TMEM (each CTA's own 128 lanes), B from shared memory.
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

}  // namespace sa
