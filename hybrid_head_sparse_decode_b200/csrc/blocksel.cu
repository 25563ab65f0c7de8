// blocksel.cu -- block-granular selection of the retrieval heads' key-token sets.
//
// The page "LycheeDecode: Accelerating Long-Context LLM Inference via
// Hybrid-Head Sparse Decoding" (paper.rainbus.top/paper/2602.04541) describes
// its decoding kernel as block-sparse; the HySparse page in the same material
// scores blocks of B = 64 positions by their largest attention score and keeps
// the k/B best blocks.  Here, for a retrieval head with n_b positions and budget
// k_b: block c covers positions [B c, min(B c + B, n_b)), its score is the
// largest logit in it (softmax is increasing, so the largest weight), and the
// max(1, floor(k_b / B)) blocks ranked first by (larger score, then lower block
// index) are taken whole.  The set is written as a membership bitmap row and/or
// an ascending index row padded with -1.
//
// A cluster of kSelCtas CTAs per (sequence, head): each reduces its share of the
// head's blocks to the order-preserving keys of their largest logits (one block
// per thread, 16-byte loads from L2, where the attention kernel just wrote
// them) and sends the keys into the shared memory of the cluster's first CTA
// (16-byte st.async stores that complete its mbarrier).  That CTA runs a radix
// select over all the keys (8-bit digits, most significant first, stopping once
// the chosen bucket holds exactly the blocks still to take) and writes the set.
// The same launch runs the combine of every head (combine_body.cuh) on its
// other CTAs: the two read disjoint data and write disjoint outputs.
#include "cluster.cuh"
#include "combine_body.cuh"
#include "common.cuh"
#include "blocksel.h"
#include "kernels.h"

namespace lychee {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kKeyThreads = 256;
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelCtas = 8;        // CTAs per (sequence, head): one cluster
static_assert(kSelCtas == kCombineSplit, "one cluster size for both roles");

__device__ __forceinline__ void head_of(const BlockSelParams& p, int pair, int& b, int& h,
                                        int& n, int& kb) {
  b = pair / p.nheads;
  h = p.heads[pair % p.nheads];
  n = min(max(p.seqlens[b], 1), p.N_max);
  kb = p.k_per_seq ? p.k_per_seq[b] : p.k;
  kb = min(min(max(kb, 1), p.k), n);
}

// Exclusive scan of one value per thread over the CTA; *total gets the sum.
__device__ __forceinline__ uint32_t cta_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const uint32_t s = wsum[w];
    before += w < warp ? s : 0u;
    all += s;
  }
  *total = all;
  __syncthreads();   // wsum is rewritten by the next scan
  return before + x - v;
}

// Before the previous kernel's results are needed: the first CTA of each
// selection cluster sets up the barrier that counts one arrival per CTA of the
// cluster (plus the bytes each sends), and the cluster learns it is set up.
__device__ __forceinline__ void block_select_prologue(uint32_t* dsm) {
  if (cluster_ctarank() == 0 && threadIdx.x == 0) {
    mbar_init(reinterpret_cast<uint64_t*>(dsm), kSelCtas);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();
}

// One CTA of the selection of (sequence, retrieval head) number `pair`, after
// block_select_prologue.  Dynamic shared memory: an mbarrier (16 bytes), then
// the block keys (in the first CTA: all of them, then per block the output
// offset of a selected block, or kFull).
__device__ __forceinline__ void block_select_body(const BlockSelParams& p, int pair, uint32_t* dsm) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t wsum[kSelWarps];
  __shared__ uint32_t bc[4];
  uint64_t* bar = reinterpret_cast<uint64_t*>(dsm);
  uint32_t* keys = dsm + 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  int b, h, n, kb;
  head_of(p, pair, b, h, n, kb);
  const int block = p.block;
  const int nblk = (n + block - 1) / block;
  const int kblk = min(max(1, kb / block), nblk);
  const size_t bh = (size_t)b * p.Hq + h;
  const float* row = p.logits + bh * p.N_max;
  // this CTA's share of the blocks: a multiple of 4 (whole 16-byte pieces)
  const int per = ((nblk + kSelCtas - 1) / kSelCtas + 3) & ~3;
  const int cb0 = min(nblk, (int)rank * per), cb1 = min(nblk, cb0 + per);
  for (int c = cb0 + tid; c < cb1; c += kSelThreads) {
    const int j0 = c * block, j1 = min(n, j0 + block);
    float mx = -INFINITY;
    int j = j0;
    if ((reinterpret_cast<uintptr_t>(row + j0) & 15u) == 0)
      for (; j + 4 <= j1; j += 4) {
        const float4 v = *reinterpret_cast<const float4*>(row + j);
        mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
      }
    for (; j < j1; ++j) mx = fmaxf(mx, row[j]);
    keys[c] = float_to_key(mx);
  }
  __syncthreads();
  cluster_wait();   // the first CTA's barrier is set up
  const uint32_t lbar = dsmem_map(smem_u32(bar), 0);
  if (rank != 0) {
    // send the keys to the same place in the first CTA
    const int nq = (cb1 - cb0 + 3) / 4;
    if (tid == 0) mbar_arrive_expect_tx_remote(lbar, (uint32_t)nq * 16u);
    for (int i = tid; i < nq; i += kSelThreads)
      st_async_v4(dsmem_map(smem_u32(keys + cb0 + 4 * i), 0),
                  *reinterpret_cast<const uint4*>(keys + cb0 + 4 * i), lbar);
    cluster_arrive_relaxed();
    cluster_wait();   // no CTA leaves while its keys may still be on their way
    return;
  }
  if (tid == 0) mbar_arrive(bar);
  mbar_wait_cluster(bar, 0u, p.err);   // every CTA's keys are here
  cluster_arrive_relaxed();

  // ---- radix select of the kblk-th largest key T
  uint32_t prefix = 0, pmask = 0, krem = (uint32_t)kblk;
  int pass = 0;
  for (; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    for (int c = tid; c < nblk; c += kSelThreads) {
      const uint32_t key = keys[c];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    // bins from the top: an inclusive sum at bin d counts the keys with digit >= d
    const int bin = 255 - tid;
    uint32_t tot = 0, incl = 0;
    if (tid < 256) {
      tot = hist[bin];
      incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t above = incl - tot;
      for (int w = 0; w < warp; ++w) above += wsum[w];
      if (above < krem && above + tot >= krem) {
        bc[0] = (uint32_t)bin;
        bc[1] = above;
        bc[2] = tot;
      }
    }
    __syncthreads();
    prefix |= (bc[0] & 255u) << shift;
    pmask |= 255u << shift;
    krem -= bc[1];
    const bool whole = bc[2] == krem;
    __syncthreads();   // bc and wsum are rewritten by the next pass
    if (whole) break;
  }
  // exact: T is the kblk-th key and krem of the blocks equal to T are taken (the
  // lowest block indices); otherwise every block whose top bits are >= the
  // chosen prefix is taken
  const bool exact = pass == 4;
  const uint32_t T = prefix;
  const uint32_t kties = exact ? krem : 0u;

  // ---- selected blocks and their output offsets, in block order
  uint32_t eq_seen = 0, sel_seen = 0;
  for (int c0 = 0; c0 < nblk; c0 += kSelThreads) {
    const int c = c0 + tid;
    const uint32_t key = c < nblk ? keys[c] : 0u;
    const bool eq = c < nblk && exact && key == T;
    uint32_t eq_tot;
    const uint32_t eq_before = eq_seen + cta_scan(eq ? 1u : 0u, wsum, &eq_tot);
    const bool sel = c < nblk && (exact ? (key > T || (eq && eq_before < kties)) : (key & pmask) >= T);
    uint32_t sel_tot;
    const uint32_t off = sel_seen + cta_scan(sel ? 1u : 0u, wsum, &sel_tot);
    if (c < nblk) keys[c] = sel ? off * (uint32_t)block : kFull;
    eq_seen += eq_tot;
    sel_seen += sel_tot;
  }
  __syncthreads();
  // ---- the set as bitmap words (blocks are whole words) and as an index row
  if (p.bitmaps) {
    uint32_t* brow = p.bitmaps + bh * p.nwords;
    const int words = (n + 31) >> 5;
    for (int w = tid; w < words; w += kSelThreads) {
      const bool in = keys[(w * 32) / block] != kFull;
      const int left = n - 32 * w;
      brow[w] = !in ? 0u : (left >= 32 ? kFull : ((1u << left) - 1u));
    }
  }
  if (p.idx_out) {
    int32_t* orow = p.idx_out + bh * p.k;
    for (int c = warp; c < nblk; c += kSelWarps) {
      const uint32_t off = keys[c];
      if (off == kFull) continue;
      const int j0 = c * block, len = min(block, n - j0);
      for (int i = lane; i < len; i += 32)
        if (off + i < (uint32_t)p.k) orow[off + i] = j0 + i;
    }
    // positions in the set: whole blocks, the tail block (if taken) cut at n_b
    const int m = (int)sel_seen * block - (keys[nblk - 1] != kFull ? nblk * block - n : 0);
    for (int t = m + tid; t < p.k; t += kSelThreads) orow[t] = -1;
  }
  cluster_wait();
}

// The selection on the first nsel CTAs (kSelCtas per head, one cluster each), the
// combine of every head on the next ncomb (the kCombineSplit CTAs of a head are
// one cluster).
template <typename T, int D>
__global__ void __launch_bounds__(kSelThreads, D >= 128 ? 2 : 1)
    block_select_combine_kernel(const __grid_constant__ BlockSelParams p,
                                const __grid_constant__ CombineParams cp, int nsel) {
  static_assert(kSelThreads == kCombThreads, "one block size for both roles");
  extern __shared__ __align__(16) uint32_t dsm[];
  unsigned char* csm = reinterpret_cast<unsigned char*>(dsm);
  pdl_launch_dependents();
  const int cta = blockIdx.x;
  if (cta < nsel) block_select_prologue(dsm);
  else combine_prologue<D>(csm);
  pdl_wait();
  if (cta < nsel) block_select_body(p, cta / kSelCtas, dsm);
  else combine_body<T, D>(cp, cta - nsel, csm);
}

template <typename T, int D>
cudaError_t launch_bsc(const BlockSelParams& p, const CombineParams& cp, cudaStream_t st) {
  auto kfn = block_select_combine_kernel<T, D>;
  static PerDeviceOnce attrs;   // per instantiation and device
  const cudaError_t ea = attrs.run([&] {
    return cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kBlockSelSmemMax);
  });
  if (ea != cudaSuccess) return ea;
  const int nsel = p.B * p.nheads * kSelCtas;
  const int ncomb = cp.B * cp.Hq * kCombineSplit;
  size_t smem = block_select_smem(p.N_max, p.block);
  if (smem > kBlockSelSmemMax) return cudaErrorInvalidValue;
  if (combine_smem_bytes<D>() > smem) smem = combine_smem_bytes<D>();
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(nsel + ncomb));
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kCombineSplit;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, p, cp, nsel);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t block_select_smem(int N_max, int block) {
  // an mbarrier, then the keys of every block (the shares rounded up to 4)
  return 16 + ((size_t)((N_max + block - 1) / block) + 4 * kSelCtas) * 4;
}

cudaError_t launch_block_select_combine(const BlockSelParams& p, const CombineParams& cp,
                                        int dtype, int D, cudaStream_t st) {
  if (p.nheads <= 0) return launch_combine(cp, dtype, D, st);
  if (dtype == 0 && D == 128) return launch_bsc<__nv_bfloat16, 128>(p, cp, st);
  if (dtype == 0 && D == 64) return launch_bsc<__nv_bfloat16, 64>(p, cp, st);
  if (dtype == 1 && D == 128) return launch_bsc<float, 128>(p, cp, st);
  if (dtype == 1 && D == 64) return launch_bsc<float, 64>(p, cp, st);
  return cudaErrorInvalidValue;
}

}  // namespace lychee
