// combine.cu -- merge of split partials into the attention output, and the
// pass-through of incoming sets for sparse heads (method steps (3)/(4) of the
// page "LycheeDecode: Accelerating Long-Context LLM Inference via Hybrid-Head
// Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// Chunk c of head h holds (m_c, l_c, a_c[d]) with m_c the largest raw dot in the
// chunk, l_c = sum_j exp((s_j - m_c)/sqrt(d)) and a_c = sum_j exp(...) V_j.  With
// M = max_c m_c and w_c = exp((m_c - M)/sqrt(d)):  O = sum_c w_c a_c / sum_c w_c l_c,
// which is softmax(q K^T / sqrt(d)) V over the head's rows.  One CTA per
// (sequence, head); the chunks are spread over the CTA's warps (each lane holds
// four output elements) and the warps' sums are added in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const __grid_constant__ CombineParams p) {
  constexpr int LPR = D / 4;            // lanes per partial row (4 elements each)
  constexpr int SLOTS = 32 / LPR;       // partial rows a warp reads at once
  constexpr int NSLOT = kWarps * SLOTS; // partial rows the CTA reads at once
  __shared__ float red[NSLOT][D + 1];   // per-slot sums; [D] holds sum of w_c l_c
  __shared__ float mred[kWarps];
  const int bh = blockIdx.x, b = bh / p.Hq, h = bh % p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_raw = p.seqlens[b];
  if (h == 0 && tid == 0) {
    if (n_raw < 1 || n_raw > p.N_max) flag_error(p.err, kErrBadSeqlen);
    if (p.k_per_seq && p.k_per_seq[b] < 1) flag_error(p.err, kErrBadBudget);
  }
  const int n = min(max(n_raw, 1), p.N_max);
  const int nc = (n + kChunk - 1) / kChunk;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)bh * p.nchunk;
  const float* pa = p.part_acc + (size_t)bh * p.nchunk * D;
  const float sl = p.scale_log2;

  float M = -INFINITY;
  for (int c = tid; c < nc; c += kThreads) {
    const float2 e = ml[c];
    if (e.y > 0.f) M = fmaxf(M, e.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) mred[warp] = M;
  __syncthreads();
  M = mred[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) M = fmaxf(M, mred[w]);

  const int slot = warp * SLOTS + lane / LPR;
  const int col = (lane % LPR) * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int c = slot; c < nc; c += NSLOT) {
      const float2 e = ml[c];
      const float4 a = *reinterpret_cast<const float4*>(pa + (size_t)c * D + col);
      const float w = e.y > 0.f ? fast_exp2((e.x - M) * sl) : 0.f;
      acc.x = fmaf(w, a.x, acc.x);
      acc.y = fmaf(w, a.y, acc.y);
      acc.z = fmaf(w, a.z, acc.z);
      acc.w = fmaf(w, a.w, acc.w);
      L = fmaf(w, e.y, L);
    }
  }
  red[slot][col + 0] = acc.x;
  red[slot][col + 1] = acc.y;
  red[slot][col + 2] = acc.z;
  red[slot][col + 3] = acc.w;
  if (lane % LPR == 0) red[slot][D] = L;
  __syncthreads();
  if (tid < D / 4) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float Ls = 0.f;
#pragma unroll
    for (int sidx = 0; sidx < NSLOT; ++sidx) {
      o.x += red[sidx][4 * tid + 0];
      o.y += red[sidx][4 * tid + 1];
      o.z += red[sidx][4 * tid + 2];
      o.w += red[sidx][4 * tid + 3];
      Ls += red[sidx][D];
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    o.x *= inv;
    o.y *= inv;
    o.z *= inv;
    o.w *= inv;
    store4<T>(reinterpret_cast<T*>(p.out) + (size_t)bh * D + 4 * tid, o);
  }

  if (bh == 0 && tid == 0 && p.counter) *p.counter = 0u;

  const bool retrieval = (p.role[h >> 5] >> (h & 31)) & 1u;
  if (!retrieval && p.idx_out && p.idx_in) {
    const int32_t* src = p.idx_in + (size_t)bh * p.k;
    int32_t* dst = p.idx_out + (size_t)bh * p.k;
    for (int t = tid; t < p.k; t += kThreads) dst[t] = src[t];
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
