// combine.cu -- merge of split partials into the attention output, and the
// pass-through of incoming sets for sparse heads (method steps (3)/(4) of the
// page "LycheeDecode: Accelerating Long-Context LLM Inference via Hybrid-Head
// Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// Chunk c of head h holds (m_c, l_c, a_c[d]) with m_c the largest raw dot in the
// chunk, l_c = sum_j exp((s_j - m_c)/sqrt(d)) and a_c = sum_j exp(...) V_j.  With
// M = max_c m_c and w_c = exp((m_c - M)/sqrt(d)):  O = sum_c w_c a_c / sum_c w_c l_c,
// which is softmax(q K^T / sqrt(d)) V over the head's rows.  One CTA per
// (sequence, head), one thread per output dimension.
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

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
__global__ void __launch_bounds__(D) combine_kernel(const __grid_constant__ CombineParams p) {
  __shared__ float wts[kChunk];   // per-chunk weight w_c (up to kChunk chunks per pass)
  __shared__ float red[D / 32];
  const int bh = blockIdx.x, b = bh / p.Hq, h = bh % p.Hq;
  const int tid = threadIdx.x;
  const int n_raw = p.seqlens[b];
  if (n_raw < 1 || n_raw > p.N_max) flag_error(p.err, kErrBadSeqlen);
  if (p.k_per_seq && p.k_per_seq[b] < 1) flag_error(p.err, kErrBadBudget);
  const int n = min(max(n_raw, 1), p.N_max);
  const int nc = (n + kChunk - 1) / kChunk;
  const float* ml = p.part_ml + (size_t)bh * p.nchunk * 2;
  const float* pa = p.part_acc + (size_t)bh * p.nchunk * D;
  const float sl = p.scale_log2;

  float M = -INFINITY;
  for (int c = tid; c < nc; c += D) {
    const float m = ml[2 * c], l = ml[2 * c + 1];
    if (l > 0.f) M = fmaxf(M, m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((tid & 31) == 0) red[tid >> 5] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);

  float acc = 0.f, L = 0.f;
  for (int c0 = 0; c0 < nc; c0 += kChunk) {
    const int cn = min(kChunk, nc - c0);
    __syncthreads();
    for (int c = tid; c < cn; c += D) {
      const float m = ml[2 * (c0 + c)], l = ml[2 * (c0 + c) + 1];
      wts[c] = (l > 0.f && M != -INFINITY) ? fast_exp2((m - M) * sl) : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < cn; ++c) {
      const float w = wts[c];
      if (w != 0.f) {
        acc = fmaf(w, pa[(size_t)(c0 + c) * D + tid], acc);
        L = fmaf(w, ml[2 * (c0 + c) + 1], L);
      }
    }
  }
  T* out = reinterpret_cast<T*>(p.out) + (size_t)bh * D;
  store_out<T>(out + tid, L > 0.f ? acc / L : 0.f);

  if (bh == 0 && tid == 0 && p.counter) *p.counter = 0u;

  const bool retrieval = (p.role[h >> 5] >> (h & 31)) & 1u;
  if (!retrieval && p.idx_out && p.idx_in) {
    const int32_t* src = p.idx_in + (size_t)bh * p.k;
    int32_t* dst = p.idx_out + (size_t)bh * p.k;
    for (int t = tid; t < p.k; t += D) dst[t] = src[t];
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int dtype, int D, cudaStream_t st) {
  const unsigned grid = (unsigned)(p.B * p.Hq);
  if (dtype == 0 && D == 128) combine_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(p);
  else if (dtype == 0 && D == 64) combine_kernel<__nv_bfloat16, 64><<<grid, 64, 0, st>>>(p);
  else if (dtype == 1 && D == 128) combine_kernel<float, 128><<<grid, 128, 0, st>>>(p);
  else if (dtype == 1 && D == 64) combine_kernel<float, 64><<<grid, 64, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lychee
