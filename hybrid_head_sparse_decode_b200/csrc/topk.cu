// topk.cu -- argsTopK of the retrieval heads' logits (method step (3) of the
// page "LycheeDecode: Accelerating Long-Context LLM Inference via Hybrid-Head
// Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// One cluster of C CTAs (16 when the GPU can schedule such clusters, else 8) per
// (sequence, retrieval head).  Each CTA owns a contiguous, word-aligned slice of
// the n_b logits and keeps them in shared memory as order-preserving uint32
// keys, so the logits are read from L2/HBM once.  An MSB-first radix select with
// 8-bit digits finds the key T of the k_b-th largest logit: each pass builds
// warp-private histograms of the next digit among the keys still matching the
// prefix, the CTA adds them up, the cluster adds the CTAs' histograms through
// distributed shared memory, and every CTA picks the same digit.  The search
// stops early when the chosen bucket holds exactly the keys still to be taken.
// The set is then every position with key > T plus the lowest-position keys == T
// up to k_b (ties go to the lower position); its positions are emitted in
// ascending order as a membership bitmap and/or an index row padded with -1.
// Softmax is strictly increasing, so selecting on logits selects the same set as
// selecting on attention weights.
#include <algorithm>

#include "combine_body.cuh"
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr size_t kSmemBudget = 200 * 1024;

// Exclusive scan of one value per thread over the CTA; *total gets the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* wsum,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kWarps ? wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += y;
    }
    wsum[lane] = t;
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? wsum[warp - 1] : 0u;
  *total = wsum[kWarps - 1];
  __syncthreads();
  return before + x - v;
}

// One CTA of the selection: CTA `cta` of cluster cta / C (its rank in the
// cluster is the hardware rank), dynamic shared memory at dsm.
template <int C>
__device__ __forceinline__ void topk_body(const TopkParams& p, int keys_cap, int wpc_cap, int cta,
                                          uint32_t* dsm) {
  uint32_t* keys = dsm;                    // [keys_cap]
  uint32_t* wa = keys + keys_cap;          // [wpc_cap] tie bits, then selected bits
  uint32_t* wb = wa + wpc_cap;             // [wpc_cap] greater bits, then output offsets
  uint32_t* whist = wb + wpc_cap;          // [kWarps][256] warp-private histograms
  __shared__ uint32_t hist[2][256];        // CTA histograms, read by the cluster
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t cta_tot[2];
  __shared__ uint32_t bc[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int pair = cta / C;
  const int b = pair / p.nheads, h = p.heads[pair % p.nheads];
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  int kb = p.k_per_seq ? p.k_per_seq[b] : p.k;
  kb = min(min(max(kb, 1), p.k), n);
  const int words = (n + 31) >> 5;
  const int wpc = (words + C - 1) / C;
  const int w0 = min(words, (int)rank * wpc), w1 = min(words, w0 + wpc);
  const int mywords = w1 - w0;
  const int pos0 = w0 * 32;
  const int npos = max(0, min(n, w1 * 32) - pos0);
  const float* row = p.logits + (size_t)(b * p.Hq + h) * p.N_max + pos0;

  const int cached = min(npos, keys_cap);
  if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
    const int nv = cached >> 2;
    for (int i = tid; i < nv; i += kThreads) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(row) + i);
      *reinterpret_cast<uint4*>(keys + 4 * i) =
          make_uint4(float_to_key(v.x), float_to_key(v.y), float_to_key(v.z), float_to_key(v.w));
    }
    for (int i = 4 * nv + tid; i < cached; i += kThreads) keys[i] = float_to_key(__ldcg(row + i));
  } else {
    for (int i = tid; i < cached; i += kThreads) keys[i] = float_to_key(__ldcg(row + i));
  }
  __syncthreads();   // the passes below read keys that other threads wrote
  auto key_at = [&](int i) -> uint32_t {
    return i < keys_cap ? keys[i] : float_to_key(__ldcg(row + i));
  };
  uint32_t* myhist = whist + warp * 256;

  // ---- radix select, 8-bit digits, most significant first
  uint32_t prefix = 0, pmask = 0;
  uint32_t krem = (uint32_t)kb;
  int pass = 0;
  for (; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const int buf = pass & 1;
    for (int i = lane; i < 256; i += 32) myhist[i] = 0u;
    __syncwarp();
    for (int i = tid; i < npos; i += kThreads) {
      const uint32_t key = key_at(i);
      if ((key & pmask) == prefix) atomicAdd(&myhist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += whist[w * 256 + tid];
      hist[buf][tid] = s;   // buffer last read in pass-2, before cluster barrier pass-1
    }
    cluster_sync();
    // cluster-wide histogram; bins enumerated from the top so that an inclusive
    // prefix sum at bin d counts the candidates whose digit is >= d
    const int bin = 255 - tid;
    uint32_t tot = 0;
    if (tid < 256) {
#pragma unroll
      for (int r2 = 0; r2 < C; ++r2) tot += dsmem_ld_u32(dsmem_addr(&hist[buf][bin], r2));
    }
    uint32_t all;
    const uint32_t above = block_exclusive_scan(tid < 256 ? tot : 0u, wsum, &all);
    if (tid < 256 && above + tot >= krem && above < krem) {
      bc[0] = (uint32_t)bin;
      bc[1] = above;
      bc[2] = tot;
    }
    __syncthreads();
    prefix |= bc[0] << shift;
    pmask |= 255u << shift;
    krem -= bc[1];
    const bool whole_bucket = bc[2] == krem;   // the same decision in every CTA
    __syncthreads();
    if (whole_bucket) break;
  }
  // exact: T is the k_b-th key and krem of the keys equal to T are taken;
  // otherwise every key whose top bits are >= the chosen prefix is taken
  const bool exact = pass == 4;
  const uint32_t T = prefix;

  // ---- compaction in position order
  for (int wl = warp; wl < mywords; wl += kWarps) {
    const int i = wl * 32 + lane;
    const bool v = i < npos;
    const uint32_t key = v ? key_at(i) : 0u;
    const uint32_t eq = __ballot_sync(kFull, v && exact && key == T);
    const uint32_t gt = __ballot_sync(kFull, v && (exact ? key > T : (key & pmask) >= T));
    if (lane == 0) {
      wa[wl] = eq;
      wb[wl] = gt;
    }
  }
  __syncthreads();
  const int wpt = (mywords + kThreads - 1) / kThreads;
  const int ta = min(mywords, tid * wpt), tb = min(mywords, ta + wpt);
  uint32_t ceq = 0, cgt = 0;
  for (int w = ta; w < tb; ++w) {
    ceq += __popc(wa[w]);
    cgt += __popc(wb[w]);
  }
  uint32_t eq_total, gt_total;
  const uint32_t eq_ex = block_exclusive_scan(ceq, wsum, &eq_total);
  (void)block_exclusive_scan(cgt, wsum, &gt_total);
  if (tid == 0) {
    cta_tot[0] = eq_total;
    cta_tot[1] = gt_total;
  }
  cluster_sync();
  const uint32_t kties = exact ? krem : 0u;
  uint32_t eq_before = 0, sel_before = 0;
  for (uint32_t r2 = 0; r2 < rank; ++r2) {
    const uint32_t e = dsmem_ld_u32(dsmem_addr(&cta_tot[0], r2));
    const uint32_t g = dsmem_ld_u32(dsmem_addr(&cta_tot[1], r2));
    const uint32_t take = kties > eq_before ? min(e, kties - eq_before) : 0u;
    sel_before += g + take;
    eq_before += e;
  }
  uint32_t run_eq = eq_before + eq_ex, csel = 0;
  uint32_t* brow = p.bitmaps ? p.bitmaps + (size_t)(b * p.Hq + h) * p.nwords + w0 : nullptr;
  for (int w = ta; w < tb; ++w) {
    const uint32_t eq = wa[w];
    const uint32_t ce = __popc(eq);
    const uint32_t allow = kties > run_eq ? min(ce, kties - run_eq) : 0u;
    uint32_t keep = eq;
    for (uint32_t c2 = ce; c2 > allow; --c2) keep &= ~(1u << (31 - __clz(keep)));
    const uint32_t sel = wb[w] | keep;
    wa[w] = sel;
    run_eq += ce;
    csel += __popc(sel);
    if (brow) brow[w] = sel;
  }
  uint32_t sel_total;
  uint32_t off = block_exclusive_scan(csel, wsum, &sel_total);
  for (int w = ta; w < tb; ++w) {
    wb[w] = off;
    off += __popc(wa[w]);
  }
  __syncthreads();
  if (p.idx_out) {
    int32_t* orow = p.idx_out + (size_t)(b * p.Hq + h) * p.k;
    for (int wl = warp; wl < mywords; wl += kWarps) {
      const uint32_t sel = wa[wl];
      if ((sel >> lane) & 1u) {
        const uint32_t o = sel_before + wb[wl] + __popc(sel & ((1u << lane) - 1u));
        if (o < (uint32_t)p.k) orow[o] = pos0 + wl * 32 + lane;
      }
    }
    if (rank == 0)
      for (int t = kb + tid; t < p.k; t += kThreads) orow[t] = -1;
  }
  cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

template <int C>
__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const __grid_constant__ TopkParams p, int keys_cap, int wpc_cap) {
  extern __shared__ __align__(16) uint32_t dsm[];
  pdl_launch_dependents();
  pdl_wait();
  topk_body<C>(p, keys_cap, wpc_cap, blockIdx.x, dsm);
}

// Top-k of the retrieval heads and the combine of all heads in one launch: the
// first ntopk CTAs (whole clusters) select, the next ncomb CTAs combine (their
// clusters never synchronise), the rest of the last cluster has nothing to do.
// The two read disjoint data (logits; partial states) and write disjoint
// outputs (sets; the attention output).
template <int C, typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    topk_combine_kernel(const __grid_constant__ TopkParams p, const __grid_constant__ CombineParams cp,
                        int keys_cap, int wpc_cap, int ntopk, int ncomb) {
  extern __shared__ __align__(16) uint32_t dsm[];
  pdl_launch_dependents();
  pdl_wait();
  const int cta = blockIdx.x;
  if (cta < ntopk) topk_body<C>(p, keys_cap, wpc_cap, cta, dsm);
  else if (cta - ntopk < ncomb) combine_body<T, D>(cp, cta - ntopk, reinterpret_cast<unsigned char*>(dsm));
}

// Launch geometry of a cluster size C for rows of up to N_max logits.
template <int C>
struct Geometry {
  int wpc_cap = 0, keys_cap = 0;
  size_t smem = 0;
  bool ok = false;
  explicit Geometry(int N_max) {
    const int words_max = (N_max + 31) / 32;
    wpc_cap = (words_max + C - 1) / C;
    const size_t fixed = (size_t)(2 * wpc_cap + kWarps * 256) * 4;
    if (fixed + 4096 > kSmemBudget) return;
    keys_cap = (int)std::min<size_t>((size_t)wpc_cap * 32, (kSmemBudget - fixed) / 4);
    smem = (size_t)keys_cap * 4 + fixed;
    ok = true;
  }
};

template <int C>
void fill_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* at, unsigned grid, size_t smem,
                 cudaStream_t st) {
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
}

template <int C>
cudaError_t set_attributes() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBudget);
  if (e == cudaSuccess && C > 8)
    e = cudaFuncSetAttribute(topk_kernel<C>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) done = true;
  return e;
}

template <int C>
cudaError_t launch_c(const TopkParams& p, cudaStream_t st) {
  const Geometry<C> g(p.N_max);
  if (!g.ok) return cudaErrorInvalidValue;
  cudaError_t e = set_attributes<C>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute at[2];
  fill_config<C>(cfg, at, (unsigned)(C * p.B * p.nheads), g.smem, st);
  e = cudaLaunchKernelEx(&cfg, topk_kernel<C>, p, g.keys_cap, g.wpc_cap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Whether clusters of 16 CTAs with this geometry can be resident (queried once
// per process for the first N_max seen, and again if a larger one fails).
bool cluster16_ok(int N_max, cudaStream_t st) {
  static int known_n = -1;
  static bool known_ok = false;
  if (known_n >= N_max) return known_ok;
  const Geometry<16> g(N_max);
  bool ok = g.ok && set_attributes<16>() == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute at[2];
    fill_config<16>(cfg, at, 16u, g.smem, st);
    cfg.numAttrs = 1;   // the occupancy query needs only the cluster shape
    int nclusters = 0;
    ok = cudaOccupancyMaxActiveClusters(&nclusters, topk_kernel<16>, &cfg) == cudaSuccess &&
         nclusters >= 1;
  }
  cudaGetLastError();   // a refused query leaves no sticky error
  known_n = N_max;
  known_ok = ok;
  return ok;
}

template <int C, typename T, int D>
cudaError_t launch_tc(const TopkParams& p, const CombineParams& cp, cudaStream_t st) {
  static_assert(kThreads == kCombThreads, "one block size for both roles");
  const Geometry<C> g(p.N_max);
  if (!g.ok) return cudaErrorInvalidValue;
  static bool done = false;
  auto kfn = topk_combine_kernel<C, T, D>;
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget);
    if (e == cudaSuccess && C > 8) e = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    done = true;
  }
  const int ntopk = C * p.B * p.nheads;
  const int ncomb = cp.B * cp.Hq * kCombineSplit;
  const int grid = (ntopk + ncomb + C - 1) / C * C;
  const size_t smem = std::max(g.smem, combine_smem_bytes<D>());
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute at[2];
  fill_config<C>(cfg, at, (unsigned)grid, smem, st);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, p, cp, g.keys_cap, g.wpc_cap, ntopk, ncomb);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_tc_d(const TopkParams& p, const CombineParams& cp, cudaStream_t st) {
  return cluster16_ok(p.N_max, st) ? launch_tc<16, T, D>(p, cp, st) : launch_tc<8, T, D>(p, cp, st);
}

}  // namespace

cudaError_t launch_topk_combine(const TopkParams& p, const CombineParams& cp, int dtype, int D,
                                cudaStream_t st) {
  if (p.nheads <= 0) return launch_combine(cp, dtype, D, st);
  if (dtype == 0 && D == 128) return launch_tc_d<__nv_bfloat16, 128>(p, cp, st);
  if (dtype == 0 && D == 64) return launch_tc_d<__nv_bfloat16, 64>(p, cp, st);
  if (dtype == 1 && D == 128) return launch_tc_d<float, 128>(p, cp, st);
  if (dtype == 1 && D == 64) return launch_tc_d<float, 64>(p, cp, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t st) {
  if (p.nheads <= 0) return cudaSuccess;
  return cluster16_ok(p.N_max, st) ? launch_c<16>(p, st) : launch_c<8>(p, st);
}

}  // namespace lychee
