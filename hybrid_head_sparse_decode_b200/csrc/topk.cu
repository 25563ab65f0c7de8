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
#include <mutex>

#include "cluster.cuh"
#include "combine_body.cuh"
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kPasses = 4;                 // 8-bit digits of a 32-bit key
constexpr int kHists = kWarps / 2;         // CTA-local histograms, one per pair of warps
constexpr size_t kSmemBudget = 200 * 1024;

// Dynamic shared memory of one selection CTA, in 32-bit words from its start:
//   bar   [kPasses] mbarriers (one per radix pass; 2 words each)
//   recv  [kPasses][C][256]  every CTA's digit histogram of each pass
//   whist [kHists][256]      this CTA's histograms, one per pair of warps
//   misc  [kMisc]            scan totals, the chosen digit, per-rank/per-warp counts
//   keys  [keys_cap]         this CTA's logits as order-preserving keys (16-byte
//                            aligned: written four at a time)
//   wa,wb [wpc_cap]          per word: keys equal to T, keys above T (bits)
constexpr int kMisc = 128;
enum : int { kMiscWtot = 0, kMiscBc = 8, kMiscRankGt = 16, kMiscRankEq = 32, kMiscWarpGt = 48,
             kMiscWarpEq = 64 };
template <int C>
struct TopkSmem {
  static constexpr int kBar = 0;
  static constexpr int kRecv = 2 * kPasses;
  static constexpr int kWhist = kRecv + kPasses * C * 256;
  static constexpr int kMiscOff = kWhist + kHists * 256;
  static constexpr int kKeys = kMiscOff + kMisc;
  static_assert(kRecv % 4 == 0 && kKeys % 4 == 0, "16-byte aligned histogram rows and keys");
  static size_t bytes(int wpc_cap, int keys_cap) {
    return (size_t)(kKeys + keys_cap + 2 * wpc_cap) * 4;
  }
};

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// The lowest `a` set bits of x (a <= popc(x)).
__device__ __forceinline__ uint32_t lowest_set_bits(uint32_t x, uint32_t a) {
  uint32_t keep = 0;
  for (uint32_t i = 0; i < a; ++i) {
    const uint32_t b = x & (0u - x);
    keep |= b;
    x ^= b;
  }
  return keep;
}

// Entries t < m of per-lane counts (gt_t: keys above T, eq_t: keys equal to T),
// in order after `eq0` keys equal to T already seen: the keys they select
// (every key above T, plus keys equal to T while fewer than kties were taken
// before them) and the keys equal to T among them.  Lanes >= n hold zeros.
__device__ __forceinline__ void prefix_take(uint32_t gt, uint32_t eq, int m, uint32_t eq0,
                                            uint32_t kties, int lane, uint32_t& sel, uint32_t& eqs) {
  const uint32_t run = eq0 + warp_inclusive_scan(eq, lane) - eq;
  const uint32_t take = kties > run ? min(eq, kties - run) : 0u;
  sel = warp_sum(lane < m ? gt + take : 0u);
  eqs = warp_sum(lane < m ? eq : 0u);
}

// Before the previous kernel's results are needed: set up the per-pass
// barriers (each expects one histogram from every CTA of the cluster), clear
// the warp histograms and announce this to the cluster.
template <int C>
__device__ __forceinline__ void topk_prologue(uint32_t* dsm) {
  using L = TopkSmem<C>;
  uint64_t* bar = reinterpret_cast<uint64_t*>(dsm + L::kBar);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) mbar_init(&bar[ps], 1);
    fence_mbar_init();
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) mbar_arrive_expect_tx(&bar[ps], C * 256 * 4);
  }
  for (int i = threadIdx.x; i < kHists * 256; i += kThreads) dsm[L::kWhist + i] = 0u;
  cluster_arrive_relaxed();
}

// One CTA of the selection: CTA `cta` of cluster cta / C (its rank in the
// cluster is the hardware rank), dynamic shared memory at dsm, after
// topk_prologue.
template <int C>
__device__ __forceinline__ void topk_body(const TopkParams& p, int keys_cap, int wpc_cap, int cta,
                                          uint32_t* dsm) {
  using L = TopkSmem<C>;
  uint64_t* bar = reinterpret_cast<uint64_t*>(dsm + L::kBar);
  uint32_t* recv = dsm + L::kRecv;
  uint32_t* whist = dsm + L::kWhist;
  uint32_t* misc = dsm + L::kMiscOff;
  uint32_t* keys = dsm + L::kKeys;
  uint32_t* wa = keys + keys_cap;
  uint32_t* wb = wa + wpc_cap;

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
  uint32_t* myhist = whist + (warp >> 1) * 256;
  const int ncache = min(npos, keys_cap);
  cluster_wait();    // every CTA's barriers are set up: histograms may be sent

  // ---- radix select, 8-bit digits, most significant first
  uint32_t prefix = 0, pmask = 0;
  uint32_t krem = (uint32_t)kb;
  // rank `warp`'s selected keys so far (warps < C; per-lane partial sums): keys
  // whose digit beat the chosen one in some pass, plus (exact) the keys equal
  // to T or (otherwise) the whole chosen bucket of the last pass
  uint32_t rk_gt = 0, rk_eq = 0;
  auto rank_counts = [&](int ps, bool last_pass, bool exact_last) {
    if (warp < C) {
      const uint32_t d = (prefix >> (24 - 8 * ps)) & 255u;
      const uint32_t* hr = recv + (ps * C + warp) * 256;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t bn = (uint32_t)(j * 32 + lane);
        if (bn > d) rk_gt += hr[bn];
      }
      if (last_pass && lane == 0) {
        if (exact_last) rk_eq += hr[d];
        else rk_gt += hr[d];
      }
    }
  };
  int pass = 0;
  for (; pass < kPasses; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll 4
    for (int i = tid; i < ncache; i += kThreads) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&myhist[(key >> shift) & 255u], 1u);
    }
    for (int i = ncache + tid; i < npos; i += kThreads) {
      const uint32_t key = key_at(i);
      if ((key & pmask) == prefix) atomicAdd(&myhist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t* rv = recv + pass * C * 256;
    if (tid < 256) {
      // this CTA's count of bin tid (the histograms are cleared for the next
      // pass as they are read), sent to slot `rank` of every CTA
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kHists; ++w) {
        s += whist[w * 256 + tid];
        whist[w * 256 + tid] = 0u;
      }
      const int q = lane & ~3;
      const uint4 v = make_uint4(__shfl_sync(kFull, s, q), __shfl_sync(kFull, s, q + 1),
                                 __shfl_sync(kFull, s, q + 2), __shfl_sync(kFull, s, q + 3));
      const uint32_t dst = smem_u32(rv + rank * 256 + (tid & ~3));
      const uint32_t bl = smem_u32(&bar[pass]);
      for (int r2 = lane & 3; r2 < C; r2 += 4) st_async_v4(dsmem_map(dst, r2), v, dsmem_map(bl, r2));
    }
    if (pass > 0) rank_counts(pass - 1, false, false);   // while the histograms travel
    mbar_wait_cluster(&bar[pass], 0u, p.err);   // all C histograms of this pass are here
    // cluster-wide histogram; bins enumerated from the top so that an inclusive
    // prefix sum at bin d counts the candidates whose digit is >= d
    const int bin = 255 - tid;
    uint32_t tot = 0, incl = 0;
    if (tid < 256) {
#pragma unroll
      for (int r2 = 0; r2 < C; ++r2) tot += rv[r2 * 256 + bin];
      incl = warp_inclusive_scan(tot, lane);
      if (lane == 31) misc[kMiscWtot + warp] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t above = incl - tot;
      for (int w = 0; w < warp; ++w) above += misc[kMiscWtot + w];
      if (above < krem && above + tot >= krem) {
        misc[kMiscBc + 0] = (uint32_t)bin;
        misc[kMiscBc + 1] = above;
        misc[kMiscBc + 2] = tot;
      }
    }
    __syncthreads();
    prefix |= (misc[kMiscBc + 0] & 255u) << shift;
    pmask |= 255u << shift;
    krem -= misc[kMiscBc + 1];
    if (misc[kMiscBc + 2] == krem) break;   // the same decision in every CTA
  }
  cluster_arrive_relaxed();  // no more histograms will arrive here (checked before exit)
  // exact: T is the k_b-th key and krem of the keys equal to T are taken;
  // otherwise every key whose top bits are >= the chosen prefix is taken
  const bool exact = pass == kPasses;
  const int last = exact ? kPasses - 1 : pass;
  const uint32_t T = prefix;
  const uint32_t kties = exact ? krem : 0u;
  rank_counts(last, true, exact);
  if (warp < C) {
    const uint32_t g = warp_sum(rk_gt);
    if (lane == 0) {
      misc[kMiscRankGt + warp] = g;
      misc[kMiscRankEq + warp] = rk_eq;
    }
  }
  // ---- this CTA's words: per warp a contiguous run, bits of keys equal to /
  // above T, and the warp's totals
  const int wpw = (mywords + kWarps - 1) / kWarps;
  const int j0 = min(mywords, warp * wpw), j1 = min(mywords, j0 + wpw);
  uint32_t ceq = 0, cgt = 0;
  for (int j = j0; j < j1; ++j) {
    const int i = j * 32 + lane;
    const bool v = i < npos;
    const uint32_t key = v ? key_at(i) : 0u;
    const uint32_t eq = __ballot_sync(kFull, v && exact && key == T);
    const uint32_t gt = __ballot_sync(kFull, v && (exact ? key > T : (key & pmask) >= T));
    if (lane == 0) {
      wa[j] = eq;
      wb[j] = gt;
    }
    ceq += __popc(eq);
    cgt += __popc(gt);
  }
  if (lane == 0) {
    misc[kMiscWarpGt + warp] = cgt;
    misc[kMiscWarpEq + warp] = ceq;
  }
  __syncthreads();

  // ---- selected keys before this warp's run: earlier ranks, then earlier warps
  uint32_t sel_r, eq_r, sel_w, eq_w;
  prefix_take(lane < C ? misc[kMiscRankGt + lane] : 0u, lane < C ? misc[kMiscRankEq + lane] : 0u,
              (int)rank, 0u, kties, lane, sel_r, eq_r);
  prefix_take(lane < kWarps ? misc[kMiscWarpGt + lane] : 0u,
              lane < kWarps ? misc[kMiscWarpEq + lane] : 0u, warp, eq_r, kties, lane, sel_w, eq_w);
  uint32_t run_eq = eq_r + eq_w, run_sel = sel_r + sel_w;

  // ---- the selected bits of each word and the output positions, 32 words at a time
  uint32_t* brow = p.bitmaps ? p.bitmaps + (size_t)(b * p.Hq + h) * p.nwords + w0 : nullptr;
  int32_t* orow = p.idx_out ? p.idx_out + (size_t)(b * p.Hq + h) * p.k : nullptr;
  for (int g0 = j0; g0 < j1; g0 += 32) {
    const int j = g0 + lane;
    const bool in = j < j1;
    const uint32_t eq = in ? wa[j] : 0u, gt = in ? wb[j] : 0u;
    const uint32_t ce = __popc(eq);
    const uint32_t ie = warp_inclusive_scan(ce, lane);
    const uint32_t r0 = run_eq + ie - ce;
    const uint32_t allow = kties > r0 ? min(ce, kties - r0) : 0u;
    const uint32_t keep = allow == ce ? eq : lowest_set_bits(eq, allow);
    const uint32_t sel = gt | keep;
    const uint32_t cs = __popc(sel);
    const uint32_t is = warp_inclusive_scan(cs, lane);
    const uint32_t off = run_sel + is - cs;
    if (in && brow) brow[j] = sel;
    if (orow) {
      const int nw = min(32, j1 - g0);
      for (int t = 0; t < nw; ++t) {
        const uint32_t s2 = __shfl_sync(kFull, sel, t);
        const uint32_t o2 = __shfl_sync(kFull, off, t);
        if ((s2 >> lane) & 1u) {
          const uint32_t o = o2 + __popc(s2 & ((1u << lane) - 1u));
          if (o < (uint32_t)p.k) orow[o] = pos0 + (g0 + t) * 32 + lane;
        }
      }
    }
    run_eq += __shfl_sync(kFull, ie, 31);
    run_sel += __shfl_sync(kFull, is, 31);
  }
  if (orow)
    for (int t = kb + (int)rank * kThreads + tid; t < p.k; t += C * kThreads) orow[t] = -1;
  cluster_wait();    // no CTA leaves while a histogram may still be on its way to it
}

// Top-k of the retrieval heads and the combine of all heads in one launch: the
// first ntopk CTAs (whole clusters) select, the next ncomb CTAs combine (each
// head's kCombineSplit CTAs are one group of a cluster, since C is a multiple
// of kCombineSplit), the rest of the last cluster only takes part in its
// cluster barriers.
// The two read disjoint data (logits; partial states) and write disjoint
// outputs (sets; the attention output).
template <int C, typename T, int D>
__global__ void __launch_bounds__(kThreads, D >= 128 ? 2 : 1)
    topk_combine_kernel(const __grid_constant__ TopkParams p, const __grid_constant__ CombineParams cp,
                        int keys_cap, int wpc_cap, int ntopk, int ncomb) {
  extern __shared__ __align__(16) uint32_t dsm[];
  pdl_launch_dependents();
  static_assert(C % kCombineSplit == 0, "a head's combine CTAs share a cluster");
  const int cta = blockIdx.x;
  unsigned char* csm = reinterpret_cast<unsigned char*>(dsm);
  if (cta < ntopk) topk_prologue<C>(dsm);
  else combine_prologue<D>(csm);
  pdl_wait();
  if (cta < ntopk) topk_body<C>(p, keys_cap, wpc_cap, cta, dsm);
  else if (cta - ntopk < ncomb) combine_body<T, D>(cp, cta - ntopk, csm);
  else combine_idle();
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
    const size_t fixed = TopkSmem<C>::bytes(wpc_cap, 0);
    if (fixed + 4096 > kSmemBudget) return;
    keys_cap = (int)std::min<size_t>((size_t)wpc_cap * 32, (kSmemBudget - fixed) / 4);
    smem = TopkSmem<C>::bytes(wpc_cap, keys_cap);
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

// Dynamic shared memory and (C = 16) the non-portable cluster size of the
// fused kernel, once per device.
template <int C, typename T, int D>
cudaError_t set_tc_attributes() {
  static PerDeviceOnce attrs;
  return attrs.run([] {
    auto kfn = topk_combine_kernel<C, T, D>;
    cudaError_t e =
        cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget);
    if (e == cudaSuccess && C > 8)
      e = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
  });
}

// Shared memory of one CTA of the fused launch: the larger of its two roles'.
template <int C, int D>
size_t tc_smem(const Geometry<C>& g) {
  return std::max(g.smem, combine_smem_bytes<D>());
}

// Whether clusters of 16 CTAs of the fused kernel, with the shared memory it is
// launched with for rows of N_max logits, can be resident on the current
// device.  Remembered per device for the largest N_max asked so far, and asked
// again for a larger one.
template <typename T, int D>
bool cluster16_ok(int N_max, cudaStream_t st) {
  static std::mutex mu;
  static int known_n[64];
  static bool known_ok[64];
  static bool init = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    for (int i = 0; i < 64; ++i) known_n[i] = -1;
    init = true;
  }
  if (known_n[dev] >= N_max) return known_ok[dev];
  const Geometry<16> g(N_max);
  bool ok = g.ok && set_tc_attributes<16, T, D>() == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute at[2];
    fill_config<16>(cfg, at, 16u, tc_smem<16, D>(g), st);
    cfg.numAttrs = 1;   // the occupancy query needs only the cluster shape
    int nclusters = 0;
    ok = cudaOccupancyMaxActiveClusters(&nclusters, topk_combine_kernel<16, T, D>, &cfg) ==
             cudaSuccess &&
         nclusters >= 1;
  }
  cudaGetLastError();   // a refused query leaves no sticky error
  known_n[dev] = N_max;
  known_ok[dev] = ok;
  return ok;
}

template <int C, typename T, int D>
cudaError_t launch_tc(const TopkParams& p, const CombineParams& cp, cudaStream_t st) {
  static_assert(kThreads == kCombThreads, "one block size for both roles");
  const Geometry<C> g(p.N_max);
  if (!g.ok) return cudaErrorInvalidValue;
  auto kfn = topk_combine_kernel<C, T, D>;
  const cudaError_t ea = set_tc_attributes<C, T, D>();
  if (ea != cudaSuccess) return ea;
  const int ntopk = C * p.B * p.nheads;
  const int ncomb = cp.B * cp.Hq * kCombineSplit;   // 0: selection only
  const int grid = (ntopk + ncomb + C - 1) / C * C;
  const size_t smem = tc_smem<C, D>(g);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute at[2];
  fill_config<C>(cfg, at, (unsigned)grid, smem, st);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, p, cp, g.keys_cap, g.wpc_cap, ntopk, ncomb);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_tc_d(const TopkParams& p, const CombineParams& cp, cudaStream_t st) {
  // With the combine in the same launch (a single layer, a stack's last layer):
  // 16 CTAs per head when the rows are long (more than 32768 logits), the GPU
  // can hold such clusters and the heads' CTAs fit one wave (two CTAs per SM);
  // else 8: many heads (a layer of retrieval heads) are then selected in one
  // wave instead of two, and short rows need fewer histogram exchanges.
  // A selection-only launch (a stack's other layers) always takes 8: it runs
  // beside the next layer's attention kernel, and a cluster of 8 needs 4 free
  // SMs at once where one of 16 needs 8 (measured: the 36-layer 128K step is
  // about 50 us shorter).
  if (cp.B == 0) return launch_tc<8, T, D>(p, cp, st);
  const long long ctas16 = 16LL * p.B * p.nheads;
  const bool one_wave = p.sms <= 0 || ctas16 <= 2LL * p.sms;
  const bool long_rows = p.N_max > 32768;
  return long_rows && one_wave && cluster16_ok<T, D>(p.N_max, st)
             ? launch_tc<16, T, D>(p, cp, st)
             : launch_tc<8, T, D>(p, cp, st);
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

}  // namespace lychee
