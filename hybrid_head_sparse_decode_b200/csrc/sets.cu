// sets.cu -- conversions between the two forms of a key-token set S (method
// steps (3)/(4) of the page "LycheeDecode: Accelerating Long-Context LLM
// Inference via Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541):
// an index row (k_b ascending positions, -1 padded) and a membership bitmap
// (bit j of word w: position 32w + j is in S).  The attention kernel reads sets
// as bitmaps so that the G heads of a KV group can be merged word by word.
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr int kThreads = 256;

// Index rows of the listed sparse heads -> bitmaps.  An entry outside [0, n_b)
// or not strictly above its predecessor sets kErrBadIndex and is skipped.
__global__ void __launch_bounds__(kThreads) build_bits_kernel(const __grid_constant__ BuildBitsParams p) {
  const int b = blockIdx.x / p.nheads, h = p.heads[blockIdx.x % p.nheads];
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  int kb = p.k_per_seq ? p.k_per_seq[b] : p.k;
  kb = min(min(max(kb, 1), p.k), n);
  const size_t bh = (size_t)b * p.Hq + h;
  uint32_t* row = p.bitmaps + bh * p.nwords;
  const int words = (n + 31) >> 5;
  for (int w = threadIdx.x; w < words; w += kThreads) row[w] = 0u;
  __syncthreads();
  const int32_t* idx = p.idx_in + bh * p.k;
  for (int t = threadIdx.x; t < kb; t += kThreads) {
    const int j = idx[t];
    const int prev = t > 0 ? idx[t - 1] : -1;
    if (j < 0 || j >= n || j <= prev) {
      flag_error(p.err, kErrBadIndex);
      continue;
    }
    atomicOr(&row[j >> 5], 1u << (j & 31));
  }
}

// Bitmaps -> index rows for every head: ascending positions, -1 padded to k.
__global__ void __launch_bounds__(kThreads) export_kernel(const __grid_constant__ ExportParams p) {
  __shared__ uint32_t wsum[kThreads / 32];
  const int bh = blockIdx.x, b = bh / p.Hq;
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const int words = (n + 31) >> 5;
  const uint32_t* row = p.bitmaps + (size_t)bh * p.nwords;
  int32_t* out = p.idx + (size_t)bh * p.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wpt = (words + kThreads - 1) / kThreads;
  const int wa = min(words, tid * wpt), wb = min(words, wa + wpt);
  const uint32_t tail = (n & 31) ? ((1u << (n & 31)) - 1u) : 0xffffffffu;
  uint32_t cnt = 0;
  for (int w = wa; w < wb; ++w) cnt += __popc(row[w] & (w == words - 1 ? tail : 0xffffffffu));
  uint32_t x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint32_t before = 0, total = 0;
  for (int i = 0; i < kThreads / 32; ++i) {
    if (i < warp) before += wsum[i];
    total += wsum[i];
  }
  uint32_t o = before + x - cnt;
  for (int w = wa; w < wb; ++w) {
    uint32_t bits = row[w] & (w == words - 1 ? tail : 0xffffffffu);
    while (bits) {
      const int j = __ffs(bits) - 1;
      bits &= bits - 1;
      if ((int)o < p.k) out[o] = w * 32 + j;
      ++o;
    }
  }
  for (int t = (int)total + tid; t < p.k; t += kThreads) out[t] = -1;
}

}  // namespace

cudaError_t launch_build_bits(const BuildBitsParams& p, cudaStream_t st) {
  if (p.nheads <= 0) return cudaSuccess;
  build_bits_kernel<<<(unsigned)(p.B * p.nheads), kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_export(const ExportParams& p, cudaStream_t st) {
  export_kernel<<<(unsigned)(p.B * p.Hq), kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace lychee
