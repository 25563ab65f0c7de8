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
// Two launches: one thread per block reduces the block to an order-preserving
// key (many CTAs per head, so the 4 n_b bytes of logits stream from L2 in
// parallel); then one CTA per (sequence, head) runs a radix select over the
// block keys in shared memory (8-bit digits, most significant first, stopping
// once the chosen bucket holds exactly the blocks still to take) and writes
// the set.
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kKeyThreads = 256;
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;

__device__ __forceinline__ void head_of(const BlockSelParams& p, int pair, int& b, int& h,
                                        int& n, int& kb) {
  b = pair / p.nheads;
  h = p.heads[pair % p.nheads];
  n = min(max(p.seqlens[b], 1), p.N_max);
  kb = p.k_per_seq ? p.k_per_seq[b] : p.k;
  kb = min(min(max(kb, 1), p.k), n);
}

// One thread per block: the key of the block's largest logit.
__global__ void __launch_bounds__(kKeyThreads) block_keys_kernel(const __grid_constant__ BlockSelParams p) {
  pdl_launch_dependents();
  pdl_wait();
  int b, h, n, kb;
  head_of(p, blockIdx.y, b, h, n, kb);
  const int nblk = (n + p.block - 1) / p.block;
  const int c = blockIdx.x * kKeyThreads + threadIdx.x;
  if (c >= nblk) return;
  const float* row = p.logits + (size_t)(b * p.Hq + h) * p.N_max;
  const int j0 = c * p.block, j1 = min(n, j0 + p.block);
  float mx = -INFINITY;
  int j = j0;
  if ((reinterpret_cast<uintptr_t>(row + j0) & 15u) == 0)
    for (; j + 4 <= j1; j += 4) {
      const float4 v = *reinterpret_cast<const float4*>(row + j);
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
  for (; j < j1; ++j) mx = fmaxf(mx, row[j]);
  p.bkeys[(size_t)(b * p.Hq + h) * p.nblk_stride + c] = float_to_key(mx);
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

// One CTA per (sequence, retrieval head): the selection and the output rows.
// keys (dynamic shared memory) hold the block keys, then per block the output
// offset of a selected block, or kFull.
__global__ void __launch_bounds__(kSelThreads, 1) block_select_kernel(const __grid_constant__ BlockSelParams p) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t wsum[kSelWarps];
  __shared__ uint32_t bc[4];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int b, h, n, kb;
  head_of(p, blockIdx.x, b, h, n, kb);
  const int block = p.block;
  const int nblk = (n + block - 1) / block;
  const int kblk = min(max(1, kb / block), nblk);
  const size_t bh = (size_t)b * p.Hq + h;
  for (int c = tid; c < nblk; c += kSelThreads) keys[c] = p.bkeys[bh * p.nblk_stride + c];

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
}

}  // namespace

size_t block_select_smem(int N_max, int block) {
  return (size_t)((N_max + block - 1) / block) * 4;
}

cudaError_t launch_block_select(const BlockSelParams& p, int stage, cudaStream_t st) {
  if (p.nheads <= 0) return cudaSuccess;
  const int nblk_max = (p.N_max + p.block - 1) / p.block;
  const size_t smem = block_select_smem(p.N_max, p.block);
  if (smem > kBlockSelSmemMax) return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(block_select_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)kBlockSelSmemMax);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaError_t e;
  if (stage == 0)
    e = launch_pdl(block_keys_kernel,
                   dim3((unsigned)((nblk_max + kKeyThreads - 1) / kKeyThreads),
                        (unsigned)(p.B * p.nheads)),
                   dim3(kKeyThreads), 0, st, p);
  else
    e = launch_pdl(block_select_kernel, dim3((unsigned)(p.B * p.nheads)), dim3(kSelThreads), smem,
                   st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lychee
