// topk.cu -- argsTopK of the retrieval heads' logits (method step (3) of the
// page "LycheeDecode: Accelerating Long-Context LLM Inference via Hybrid-Head
// Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// One cluster of kCluster CTAs per (sequence, retrieval head).  Each CTA owns a
// contiguous, word-aligned slice of the n_b logits and keeps them in shared
// memory as order-preserving uint32 keys, so the logits are read from L2/HBM
// once.  An MSB-first radix select with 8-bit digits (4 passes) finds the key T
// of the k_b-th largest logit: each pass builds a per-CTA histogram of the next
// digit among the keys still matching the prefix (warp-aggregated shared
// atomics), the cluster sums the histograms through distributed shared memory,
// and every CTA picks the same digit.  The set is then every position with key
// > T plus the lowest-position keys == T up to k_b (ties go to the lower
// position); its positions are emitted in ascending order as a membership
// bitmap and/or an index row padded with -1.  Softmax is strictly increasing, so
// selecting on logits selects the same set as selecting on attention weights.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr size_t kSmemBudget = 220 * 1024;

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

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    topk_kernel(const __grid_constant__ TopkParams p, int keys_cap, int wpc_cap) {
  extern __shared__ __align__(16) uint32_t dsm[];
  uint32_t* keys = dsm;                    // [keys_cap]
  uint32_t* wa = keys + keys_cap;          // [wpc_cap] tie bits, then selected bits
  uint32_t* wb = wa + wpc_cap;             // [wpc_cap] greater bits, then output offsets
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t cta_tot[2];
  __shared__ uint32_t bc[2];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x / kCluster;
  const int b = pair / p.nheads, h = p.heads[pair % p.nheads];
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  int kb = p.k_per_seq ? p.k_per_seq[b] : p.k;
  kb = min(min(max(kb, 1), p.k), n);
  const int words = (n + 31) >> 5;
  const int wpc = (words + kCluster - 1) / kCluster;
  const int w0 = min(words, (int)rank * wpc), w1 = min(words, w0 + wpc);
  const int mywords = w1 - w0;
  const int pos0 = w0 * 32;
  const int npos = max(0, min(n, w1 * 32) - pos0);
  const float* row = p.logits + (size_t)(b * p.Hq + h) * p.N_max + pos0;

  const int cached = min(npos, keys_cap);
  for (int i = tid; i < cached; i += kThreads) keys[i] = float_to_key(row[i]);
  for (int i = tid; i < 512; i += kThreads) (&hist[0][0])[i] = 0u;
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t {
    return i < keys_cap ? keys[i] : float_to_key(__ldg(row + i));
  };

  // ---- radix select: 4 passes of 8 bits, most significant first
  uint32_t prefix = 0, pmask = 0;
  uint32_t krem = (uint32_t)kb;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const int buf = pass & 1;
    if (pass >= 2) {
      // buffer last read in pass-2; every CTA passed the cluster barrier of pass-1
      for (int i = tid; i < 256; i += kThreads) hist[buf][i] = 0u;
      __syncthreads();
    }
    for (int base = 0; base < npos; base += kThreads) {
      const int i = base + tid;
      uint32_t key = 0;
      bool act = false;
      if (i < npos) {
        key = key_at(i);
        act = (key & pmask) == prefix;
      }
      const uint32_t am = __ballot_sync(kFull, act);
      if (act) {
        const uint32_t bin = (key >> shift) & 255u;
        const uint32_t peers = __match_any_sync(am, bin);
        if (__ffs(peers) - 1 == lane) atomicAdd(&hist[buf][bin], (uint32_t)__popc(peers));
      }
    }
    cluster_sync();
    // cluster-wide histogram; bins enumerated from the top so that an inclusive
    // prefix sum at bin d counts the candidates whose digit is >= d
    const int bin = 255 - tid;
    uint32_t tot = 0;
    if (tid < 256)
      for (int r2 = 0; r2 < kCluster; ++r2) tot += dsmem_ld_u32(dsmem_addr(&hist[buf][bin], r2));
    uint32_t all;
    const uint32_t above = block_exclusive_scan(tid < 256 ? tot : 0u, wsum, &all);
    if (tid < 256 && above + tot >= krem && above < krem) {
      bc[0] = (uint32_t)bin;
      bc[1] = above;
    }
    __syncthreads();
    prefix |= bc[0] << shift;
    pmask |= 255u << shift;
    krem -= bc[1];
    __syncthreads();
  }
  const uint32_t T = prefix;  // key of the k_b-th largest logit; krem ties are taken

  // ---- compaction in position order
  for (int wl = warp; wl < mywords; wl += kWarps) {
    const int i = wl * 32 + lane;
    const bool v = i < npos;
    const uint32_t key = v ? key_at(i) : 0u;
    const uint32_t eq = __ballot_sync(kFull, v && key == T);
    const uint32_t gt = __ballot_sync(kFull, v && key > T);
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
  uint32_t eq_before = 0, sel_before = 0;
  for (uint32_t r2 = 0; r2 < rank; ++r2) {
    const uint32_t e = dsmem_ld_u32(dsmem_addr(&cta_tot[0], r2));
    const uint32_t g = dsmem_ld_u32(dsmem_addr(&cta_tot[1], r2));
    const uint32_t take = krem > eq_before ? min(e, krem - eq_before) : 0u;
    sel_before += g + take;
    eq_before += e;
  }
  uint32_t run_eq = eq_before + eq_ex, csel = 0;
  uint32_t* brow = p.bitmaps ? p.bitmaps + (size_t)(b * p.Hq + h) * p.nwords + w0 : nullptr;
  for (int w = ta; w < tb; ++w) {
    const uint32_t eq = wa[w];
    const uint32_t ce = __popc(eq);
    const uint32_t allow = krem > run_eq ? min(ce, krem - run_eq) : 0u;
    uint32_t keep = eq;
    for (uint32_t c = ce; c > allow; --c) keep &= ~(1u << (31 - __clz(keep)));
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

}  // namespace

cudaError_t launch_topk(const TopkParams& p, cudaStream_t st) {
  if (p.nheads <= 0) return cudaSuccess;
  const int words_max = (p.N_max + 31) / 32;
  const int wpc_cap = (words_max + kCluster - 1) / kCluster;
  const size_t bits_bytes = (size_t)2 * wpc_cap * 4;
  if (bits_bytes + 4096 > kSmemBudget) return cudaErrorInvalidValue;
  const int keys_cap = (int)std::min<size_t>((size_t)wpc_cap * 32, (kSmemBudget - bits_bytes) / 4);
  const size_t smem = ((size_t)keys_cap + 2 * wpc_cap) * 4;
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBudget);
    if (e != cudaSuccess) return e;
    attr = kSmemBudget;
  }
  const long long grid = (long long)kCluster * p.B * p.nheads;
  topk_kernel<<<(unsigned)grid, kThreads, smem, st>>>(p, keys_cap, wpc_cap);
  return cudaGetLastError();
}

}  // namespace lychee
