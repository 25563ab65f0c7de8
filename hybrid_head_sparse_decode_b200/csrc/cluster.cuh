// cluster.cuh -- exchanges between the CTAs of a thread-block cluster beyond
// the plain barrier of common.cuh: split cluster barriers, 16-byte stores into
// another CTA's shared memory that complete on its mbarrier (st.async), and
// bounded cluster-scope waits on such an mbarrier.  Used by the top-k.
#pragma once

#include "common.cuh"

namespace lychee {

// The same shared-window offset (a shared::cta address) in CTA `rank`'s window.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(local), "r"(rank));
  return out;
}

// Split cluster barrier: every thread of every CTA of the cluster arrives, and
// a later wait returns once all have.  The relaxed arrival does not order this
// thread's earlier memory accesses (for a barrier that only marks progress, or
// after fence_mbar_init).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16-byte store into another CTA's shared memory (both addresses from
// dsmem_map); its bytes count as transaction bytes on that CTA's mbarrier.
__device__ __forceinline__ void st_async_v4(uint32_t remote, uint4 v, uint32_t remote_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, "
      "[%5];" ::"r"(remote),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(remote_bar)
      : "memory");
}

// Arrival on another CTA's mbarrier (address from dsmem_map) that also raises
// its expected transaction bytes by `bytes`.
__device__ __forceinline__ void mbar_arrive_expect_tx_remote(uint32_t remote_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   remote_bar),
               "r"(bytes)
               : "memory");
}

// Bounded wait on a local mbarrier whose transaction bytes come from other CTAs
// of the cluster: acquire at cluster scope, so their stores are visible after.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity,
                                                      uint32_t hint_ns = 1000000u) {
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
// Gives up after kWaitLimitNs and sets kErrTimeout (the caller carries on with
// whatever arrived; every later access stays within its buffers).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      flag_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

}  // namespace lychee
