// combine.cu -- merge of split partials into the attention output (method steps
// (3)/(4) of the page "LycheeDecode: Accelerating Long-Context LLM Inference via
// Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// Chunk c of head h holds (m_c, l_c, a_c[d]) with m_c the largest raw dot in the
// chunk, l_c = sum_j exp((s_j - m_c)/sqrt(d)) and a_c = sum_j exp(...) V_j.  With
// M = max_c m_c and w_c = exp((m_c - M)/sqrt(d)):  O = sum_c w_c a_c / sum_c w_c l_c,
// which is softmax(q K^T / sqrt(d)) V over the head's rows.
//
// One CTA of 512 threads per (sequence, head).  Each lane owns four of the d
// elements of one "slot"; a slot walks every NS-th chunk keeping its own running
// maximum (rescaling its sums when the maximum grows), so all loads of a slot are
// independent and in flight together.  The slots are then merged in a fixed
// order in shared memory: the result does not depend on scheduling.
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) {
  *p = v;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const __grid_constant__ CombineParams p) {
  constexpr int LPR = D / 4;             // lanes per partial row
  constexpr int SLOTS = 32 / LPR;        // partial rows a warp reads at once
  constexpr int NS = kWarps * SLOTS;     // slots of the CTA
  constexpr int RS = D + 4;              // smem row: acc[D], m, l, pad
  __shared__ __align__(16) float red[NS * RS];
  const int bh = blockIdx.x, b = bh / p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const int nc = (n + kChunk - 1) / kChunk;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)bh * p.nchunk;
  const float* pa = p.part_acc + (size_t)bh * p.nchunk * D;
  const float sl = p.scale_log2;

  const int slot = warp * SLOTS + lane / LPR;
  const int col = (lane % LPR) * 4;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int c = slot; c < nc; c += NS) {
    const float2 e = ml[c];
    const float4 a = *reinterpret_cast<const float4*>(pa + (size_t)c * D + col);
    if (e.y > 0.f) {
      if (e.x > m) {
        const float r = fast_exp2((m - e.x) * sl);   // 0 while m is -inf
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
        l *= r;
        m = e.x;
      }
      const float w = fast_exp2((e.x - m) * sl);
      acc.x = fmaf(w, a.x, acc.x);
      acc.y = fmaf(w, a.y, acc.y);
      acc.z = fmaf(w, a.z, acc.z);
      acc.w = fmaf(w, a.w, acc.w);
      l = fmaf(w, e.y, l);
    }
  }
  float* row = red + slot * RS;
  *reinterpret_cast<float4*>(row + col) = acc;
  if (col == 0) {
    row[D] = m;
    row[D + 1] = l;
  }
  __syncthreads();
  if (tid < D) {
    float M = -INFINITY;
    for (int s2 = 0; s2 < NS; ++s2) M = fmaxf(M, red[s2 * RS + D]);
    float A = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < NS; ++s2) {
        const float ms = red[s2 * RS + D];
        const float w = ms == -INFINITY ? 0.f : fast_exp2((ms - M) * sl);
        A = fmaf(w, red[s2 * RS + tid], A);
        L = fmaf(w, red[s2 * RS + D + 1], L);
      }
    }
    store_out<T>(reinterpret_cast<T*>(p.out) + (size_t)bh * D + tid, L > 0.f ? A / L : 0.f);
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int dtype, int D, cudaStream_t st) {
  const unsigned grid = (unsigned)(p.B * p.Hq);
  if (dtype == 0 && D == 128) combine_kernel<__nv_bfloat16, 128><<<grid, kThreads, 0, st>>>(p);
  else if (dtype == 0 && D == 64) combine_kernel<__nv_bfloat16, 64><<<grid, kThreads, 0, st>>>(p);
  else if (dtype == 1 && D == 128) combine_kernel<float, 128><<<grid, kThreads, 0, st>>>(p);
  else if (dtype == 1 && D == 64) combine_kernel<float, 64><<<grid, kThreads, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lychee
