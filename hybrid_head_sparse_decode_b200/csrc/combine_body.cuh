// combine_body.cuh -- one CTA of the merge of attention partial states into
// the output (see combine.cu); shared by the combine kernel and the fused
// top-k + combine launch (topk.cu).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lychee {

constexpr int kCombThreads = 512;
constexpr int kCombWarps = kCombThreads / 32;

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

constexpr int kBatch = 4;

// Merge one state (e = (m, l), a = four elements of acc) into running sums.
__device__ __forceinline__ void absorb(float2 e, float4 a, float sl, float& m, float& l,
                                       float4& acc) {
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

// Shared memory one combine CTA uses (16-byte aligned start).
template <int D>
constexpr size_t combine_smem_bytes() {
  return (size_t)(kCombWarps * (32 / (D / 4)) * (D + 4)) * 4 + kCombThreads * kPartSlots * 2 +
         kCombWarps * 4 + 16;
}

// One combine CTA: `cta` numbers the CTA among all combine CTAs, `sm` is its
// shared memory (combine_smem_bytes<D>() bytes).  kCombThreads threads.
template <typename T, int D>
__device__ __forceinline__ void combine_body(const CombineParams& p, int cta, unsigned char* sm) {
  constexpr int kThreads = kCombThreads, kWarps = kCombWarps;
  constexpr int LPR = D / 4;             // lanes per state row
  constexpr int SLOTS = 32 / LPR;        // state rows a warp reads at once
  constexpr int NS = kWarps * SLOTS;     // slots of the CTA
  constexpr int RS = D + 4;              // smem row: acc[D], m, l, pad
  float* red = reinterpret_cast<float*>(sm);                                     // [NS * RS]
  uint16_t* slist = reinterpret_cast<uint16_t*>(sm + NS * RS * 4);               // (chunk, state)
  int* wsum = reinterpret_cast<int*>(sm + NS * RS * 4 + kThreads * kPartSlots * 2);
  int& is_last = wsum[kWarps];
  const int bh = cta / kCombineSplit, sp = cta % kCombineSplit;
  const int b = bh / p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const int nc = (n + kChunk - 1) / kChunk;
  const int cps = (nc + kCombineSplit - 1) / kCombineSplit;
  const int c_lo = min(nc, sp * cps), c_hi = min(nc, c_lo + cps);
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)bh * p.nchunk * kPartSlots;
  const float* pa = p.part_acc + (size_t)bh * p.nchunk * kPartSlots * D;
  const int32_t* pn = p.part_n + (size_t)bh * p.nchunk;
  const float sl = p.scale_log2;

  const int slot = warp * SLOTS + lane / LPR;
  const int col = (lane % LPR) * 4;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = c_lo; c0 < c_hi; c0 += kThreads) {
    // list this block's states in order
    const int ns = c0 + tid < c_hi ? min(max(pn[c0 + tid], 0), kPartSlots) : 0;
    int incl = ns;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int v = wsum[w];
      before += w < warp ? v : 0;
      tot += v;
    }
    const int excl = before + incl - ns;
    for (int j = 0; j < ns; ++j) slist[excl + j] = (uint16_t)(tid * kPartSlots + j);
    __syncthreads();
    for (int st0 = slot; st0 < tot; st0 += NS * kBatch) {
      float2 e[kBatch];
      float4 a[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int st = st0 + q * NS;
        e[q] = make_float2(-INFINITY, 0.f);
        a[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (st < tot) {
          const int e16 = slist[st];
          const size_t si = (size_t)(c0 + e16 / kPartSlots) * kPartSlots + e16 % kPartSlots;
          e[q] = ml[si];
          a[q] = *reinterpret_cast<const float4*>(pa + si * D + col);
        }
      }
#pragma unroll
      for (int q = 0; q < kBatch; ++q) absorb(e[q], a[q], sl, m, l, acc);
    }
    __syncthreads();   // wsum and the list are rewritten for the next block
  }
  float* row = red + slot * RS;
  *reinterpret_cast<float4*>(row + col) = acc;
  if (col == 0) {
    row[D] = m;
    row[D + 1] = l;
  }
  __syncthreads();
  // this CTA's state, merged over the slots in order
  float* st = p.part2 + (size_t)cta * RS;
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
    st[tid] = A;
    if (tid == 0) {
      st[D] = M;
      st[D + 1] = L;
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    is_last = atomicAdd(&p.ccnt[bh], 1u) == kCombineSplit - 1;
  }
  __syncthreads();
  if (!is_last) return;
  // the head's last CTA: merge the kCombineSplit states in order
  __threadfence();
  if (tid < D) {
    const float* s0 = p.part2 + (size_t)bh * kCombineSplit * RS;
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kCombineSplit; ++k) M = fmaxf(M, __ldcg(s0 + k * RS + D));
    float A = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int k = 0; k < kCombineSplit; ++k) {
        const float ms = __ldcg(s0 + k * RS + D);
        const float w = ms == -INFINITY ? 0.f : fast_exp2((ms - M) * sl);
        A = fmaf(w, __ldcg(s0 + k * RS + tid), A);
        L = fmaf(w, __ldcg(s0 + k * RS + D + 1), L);
      }
    }
    store_out<T>(reinterpret_cast<T*>(p.out) + (size_t)bh * D + tid, L > 0.f ? A / L : 0.f);
  }
  if (tid == 0) p.ccnt[bh] = 0u;   // ready for the next launch
}


}  // namespace lychee
