// common.cuh -- device helpers shared by the libychee kernels (sm_100a).
//
// Everything here is plain inline PTX for the Hopper/Blackwell asynchronous
// copy machinery (mbarrier, 1-D bulk copies into shared memory, cluster
// barriers and distributed shared memory) plus the workspace layout.  No TMA
// copy here uses cluster multicast, and every source address is this GPU's own
// global memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace lychee {

// ---- device error word (workspace header) ---------------------------------
enum : uint32_t {
  kErrBadIndex = 1u,    // incoming index out of range or not strictly ascending
  kErrBadSeqlen = 2u,   // n_b outside [1, N_max] (clamped)
  kErrBadBudget = 4u,   // k_per_seq[b] < 1 (clamped to 1)
  kErrTimeout = 8u,     // a pipeline wait gave up
};

// Workspace header: 256 bytes at offset 0.
struct WsHeader {
  uint32_t err;          // error bits (above)
  uint32_t pad0[15];
  uint32_t counters[48]; // per-launch work counters (zeroed at the start of a call)
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kChunk = 960;           // positions per attention work item, at most (30 words)
constexpr int kChunkMin = 768;        // ... and at least (the host picks one per launch),
constexpr int kChunkSmall = 128;      // ... or this for a layer with fewer K/V rows than
constexpr long long kSmallLayerRows = 256LL * kChunkMin;   // this (too few for every SM)
constexpr int kPartSlots = 12;        // partial states per (sequence, head, chunk): one per warp
constexpr int kMaxHq = 128;           // query heads supported
constexpr int kMaxWindow = 1024;      // rows of a sparse head's sliding-window ring, at most
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: a wait this long is a fault

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void flag_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

// ---- shared-memory addresses -----------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// One bounded wait: the thread may be suspended until the phase completes or
// about `hint_ns` elapse (a hint to the hardware), so waiting warps do not spin.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity,
                                              uint32_t hint_ns = 1000000u) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after
// limit_ns, sets kErrTimeout and returns false; the caller then leaves.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) {
      flag_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

// ---- 16-byte asynchronous copies global -> shared (cp.async, L2 only) -------
// The plain three-operand form: a fourth operand would be read as the source
// size of a zero-filling copy.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// The mbarrier's pending count is raised by one now and lowered again when all
// of this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- 1-D bulk copy global -> shared (TMA, no tensor map, no multicast) ------
// dst and src 16-byte aligned, bytes a multiple of 16.  Completion is signalled
// as transaction bytes on `bar`.  The L2 policy marks the streamed cache rows
// evict-first: they are read once per step.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- row gather through a tensor map (TMA tile::gather4, no multicast) ----------
// The tensor map describes a 2-D array of rows (inner dimension: the row's
// elements) with a box one row high and one full row wide.  One instruction
// copies rows y0..y3 (any order, repeats allowed), columns from x (a multiple
// of 16 bytes; 0 here), into four consecutive box-sized slots at dst (128-byte
// aligned).  Completion is signalled as transaction bytes on `bar`.
__device__ __forceinline__ void tma_gather4(void* dst, const void* tmap, int x, int y0, int y1,
                                            int y2, int y3, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- 3-D tiled load through a tensor map (TMA, no multicast) ----------------------
// Copies the box at coordinates (x, y, z) (x innermost, x * element size a
// multiple of 16 bytes) to dst, in the map's shared-memory layout (with a
// 128-byte swizzle: dst 1024-byte aligned); elements outside the tensor read as
// zero.  Completion is signalled as the box's bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int x, int y, int z,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// ---- four 8x8 matrices of 16-bit elements from shared memory ------------------------
// Lanes 8i .. 8i + 7 give the addresses of the 8 rows (16 bytes each) of matrix
// i; lane 4r + c receives, of each matrix, the elements at columns 2c and
// 2c + 1 of row r.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// ---- four 8x8 matrices of 16-bit elements from shared memory, transposed ------------
// Lanes 8i .. 8i + 7 give the addresses of the 8 rows (16 bytes each) of matrix
// i; lane 4r + c receives, of each matrix, the elements at rows 2c and 2c + 1 of
// column r (the lower half of the register holding row 2c).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// ---- programmatic dependent launch -------------------------------------------------
// Every kernel of the library lets the next kernel of its stream start launching
// at once (its CTAs become resident as SMs free up) and, before touching any
// memory, waits until the previous kernel of the stream has completed and its
// writes are visible.  With the launch attribute below this hides the launch
// gap between dependent kernels; without it both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---- named barriers (a subset of the CTA's warps) ------------------------------
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- clusters / distributed shared memory ---------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Address of `p` (a shared variable of this CTA) in the shared window of CTA
// `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}

__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// ---- numeric helpers --------------------------------------------------------------
// 2^x on the special-function unit (PTX ex2.approx.ftz; its error is orders of
// magnitude below the output tolerances; inputs here are <= 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map of an fp32 value to uint32 (larger float -> larger key).
// -0.0 is folded onto +0.0 so that equal values compare equal.
__device__ __forceinline__ uint32_t float_to_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// bf16x2 in one 32-bit word -> two fp32 (exact widening).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ---- per-device one-time host work ----------------------------------------------
// Kernel attributes (dynamic shared memory, cluster sizes) are per device.  A
// PerDeviceOnce remembers, per device ordinal below 64, that its work succeeded
// on that device; callers from several host threads may both run it the first
// time (the work is idempotent), never neither.  Devices 64 and up repeat the
// work on every call.
class PerDeviceOnce {
 public:
  template <typename F>
  cudaError_t run(F&& work) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return work();
    const uint64_t bit = 1ull << dev;
    if (done_.load(std::memory_order_acquire) & bit) return cudaSuccess;
    const cudaError_t w = work();
    if (w == cudaSuccess) done_.fetch_or(bit, std::memory_order_acq_rel);
    return w;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// Launch with programmatic stream serialization (see pdl_wait above).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace lychee
