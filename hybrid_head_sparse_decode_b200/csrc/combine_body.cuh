// combine_body.cuh -- one CTA of the merge of attention partial states into
// the output (see combine.cu); shared by the combine kernel and the fused
// top-k + combine launch (topk.cu).
#pragma once

#include "cluster.cuh"
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

constexpr int kBatch = 5;

// ---- the sliding-window branch of a sparse head -------------------------------------
// Page "HySparse: A Hybrid Sparse Attention Architecture with Oracle Token
// Selection and KV Cache Sharing" (paperlayer.ai/abs/2602.03560v1),
// Methodology: a sparse layer fuses its sparse branch with a local
// sliding-window branch (window 128, its own cache) through sigmoid gating.
// Here the window branch of sparse head h attends to the min(window, n_b) rows
// in use of its KV group's window ring (position j lives in row j % window; the
// order of the rows does not matter to softmax), and the head's output is
// s * O_sparse + (1 - s) * O_window with s = sigmoid(gate logit).

// Shared memory of window_out, in floats: q, the row scores, two reduction slots.
template <int D>
constexpr int window_smem_floats() {
  return D + kMaxWindow + 32;
}

template <typename T>
__device__ __forceinline__ float elem_to_float(const T* p, int i);
template <>
__device__ __forceinline__ float elem_to_float<__nv_bfloat16>(const __nv_bfloat16* p, int i) {
  return __bfloat162float(p[i]);
}
template <>
__device__ __forceinline__ float elem_to_float<float>(const float* p, int i) {
  return p[i];
}

// Dot product of the fp32 vector sq[0 .. D) with row r (16-byte loads).
template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* sq, const T* r) {
  const uint4* v = reinterpret_cast<const uint4*>(r);
  float acc = 0.f;
  if constexpr (sizeof(T) == 2) {
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
      const uint4 w = __ldg(v + c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = bf16x2_to_float2(ws[e]);
        acc = fmaf(sq[8 * c + 2 * e], f.x, acc);
        acc = fmaf(sq[8 * c + 2 * e + 1], f.y, acc);
      }
    }
  } else {
#pragma unroll 4
    for (int c = 0; c < D / 4; ++c) {
      const uint4 w = __ldg(v + c);
      acc = fmaf(sq[4 * c], __uint_as_float(w.x), acc);
      acc = fmaf(sq[4 * c + 1], __uint_as_float(w.y), acc);
      acc = fmaf(sq[4 * c + 2], __uint_as_float(w.z), acc);
      acc = fmaf(sq[4 * c + 3], __uint_as_float(w.w), acc);
    }
  }
  return acc;
}

// Whether head h of a layer gets the window branch.
__device__ __forceinline__ bool window_on(const WindowParams& w, int h) {
  return w.k != nullptr && !((w.role[h >> 5] >> (h & 31)) & 1u);
}

// The window branch's output element threadIdx.x (< D) of head bh = b * Hq + h
// with n_b = n, computed by every thread of the CTA (a call the whole CTA makes
// together); sm: window_smem_floats<D>() floats of shared memory.  Scores are
// fp32 sums of exact products, the softmax and the weighted sum fp32, in a
// fixed order.
template <typename T, int D>
__device__ __forceinline__ float window_out(const WindowParams& w, int bh, int Hq, int n,
                                            float sl, float* sm) {
  float* sq = sm;
  float* ss = sm + D;
  float* red = ss + kMaxWindow;
  const int b = bh / Hq, h = bh % Hq, g = h / (Hq / w.Hkv);
  const T* qr = reinterpret_cast<const T*>(w.q) + (size_t)bh * D;
  const size_t ring = ((size_t)b * w.Hkv + g) * (size_t)w.window * D;
  const T* K = reinterpret_cast<const T*>(w.k) + ring;
  const T* V = reinterpret_cast<const T*>(w.v) + ring;
  const int rows = min(min(w.window, n), kMaxWindow);
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < D; i += blockDim.x) sq[i] = elem_to_float<T>(qr, i);
  __syncthreads();
  for (int r = tid; r < rows; r += blockDim.x) ss[r] = dot_row<T, D>(sq, K + (size_t)r * D);
  __syncthreads();
  if (tid < 32) {
    float m = -INFINITY;
    for (int r = lane; r < rows; r += 32) m = fmaxf(m, ss[r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[0] = m;
  }
  __syncthreads();
  const float m = red[0];
  for (int r = tid; r < rows; r += blockDim.x) ss[r] = fast_exp2((ss[r] - m) * sl);
  __syncthreads();
  if (tid < 32) {
    float l = 0.f;
    for (int r = lane; r < rows; r += 32) l += ss[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) red[1] = l;
  }
  __syncthreads();
  float o = 0.f;
  if (tid < D) {
    for (int r = 0; r < rows; ++r) o = fmaf(ss[r], elem_to_float<T>(V + (size_t)r * D, tid), o);
    o /= red[1];
  }
  __syncthreads();   // sm is reused by the caller
  return o;
}

// s * o_sparse + (1 - s) * o_window with s = sigmoid(g).
__device__ __forceinline__ float gate_fuse(float o_sparse, float o_window, float g) {
  const float s = 1.f / (1.f + expf(-g));
  return s * o_sparse + (1.f - s) * o_window;
}

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

constexpr int kCombineSplit = 8;   // combine CTAs per (sequence, head): one group of a cluster

// Shared memory of one combine CTA, in bytes from its (16-byte aligned) start:
//   bar   one mbarrier (8 bytes, padded to 16)
//   recv  [kCombineSplit][D + 4] floats: the head's CTA states (leader CTA only)
//   red   [NS][D + 4] floats: this CTA's slot states, then its own state
//   slist [kCombThreads * kPartSlots] u16: the states of a block of chunks, in order
//         (then, in the leader, the window branch's scratch)
//   wsum  [kCombWarps + 1] ints
template <int D>
struct CombineSmem {
  static constexpr int RS = D + 4;                       // state row: acc[D], m, l, pad
  static constexpr int NS = kCombWarps * (32 / (D / 4)); // slots of the CTA
  static constexpr size_t kRecv = 16;
  static constexpr size_t kRed = kRecv + (size_t)kCombineSplit * RS * 4;
  static constexpr size_t kSlist = kRed + (size_t)(NS + 1) * RS * 4;
  static constexpr size_t kWsum = kSlist + (size_t)kCombThreads * kPartSlots * 2;
  static constexpr size_t kBytes = kWsum + (kCombWarps + 1) * 4;
  static_assert(kRed % 16 == 0 && kSlist % 16 == 0 && (RS * 4) % 16 == 0, "16-byte rows");
  static_assert((size_t)kCombThreads * kPartSlots * 2 >= (size_t)window_smem_floats<D>() * 4,
                "the window branch's scratch fits the state list");
};
template <int D>
constexpr size_t combine_smem_bytes() {
  return CombineSmem<D>::kBytes;
}

// Before the previous kernel's results are needed: the CTA's mbarrier expects
// the states of the other kCombineSplit - 1 CTAs of its head (only the head's
// first CTA, its leader, receives any), and the cluster learns it is set up.
// Every CTA of a launch whose clusters hold combine CTAs runs this, idle ones too.
template <int D>
__device__ __forceinline__ void combine_prologue(unsigned char* sm) {
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, (kCombineSplit - 1) * CombineSmem<D>::RS * 4);
  }
  cluster_arrive_relaxed();
}

// The two remaining cluster barriers of a CTA that has no state to combine.
__device__ __forceinline__ void combine_idle() {
  cluster_wait();
  cluster_arrive_relaxed();
  cluster_wait();
}

// One combine CTA, after combine_prologue: `cta` numbers the CTA among all
// combine CTAs (the kCombineSplit CTAs of a head are consecutive and start a
// group of the cluster), `sm` is its shared memory (combine_smem_bytes<D>()
// bytes).  kCombThreads threads.
template <typename T, int D>
__device__ __forceinline__ void combine_body(const CombineParams& p, int cta, unsigned char* sm) {
  using L = CombineSmem<D>;
  constexpr int kThreads = kCombThreads, kWarps = kCombWarps;
  constexpr int LPR = D / 4;             // lanes per state row
  constexpr int SLOTS = 32 / LPR;        // state rows a warp reads at once
  constexpr int NS = L::NS;
  constexpr int RS = L::RS;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  float* recv = reinterpret_cast<float*>(sm + L::kRecv);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  uint16_t* slist = reinterpret_cast<uint16_t*>(sm + L::kSlist);
  int* wsum = reinterpret_cast<int*>(sm + L::kWsum);
  const int bh = cta / kCombineSplit, sp = cta % kCombineSplit;
  const int b = bh / p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const int nc = (n + p.chunk - 1) / p.chunk;
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
  // this CTA's state, merged over the slots in order: the leader keeps it in
  // its first receive row, the others stage it for sending
  float* mine = sp == 0 ? recv : red + NS * RS;
  if (tid < D) {
    float M = -INFINITY;
    for (int s2 = 0; s2 < NS; ++s2) M = fmaxf(M, red[s2 * RS + D]);
    float A = 0.f, Lsum = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < NS; ++s2) {
        const float ms = red[s2 * RS + D];
        const float w = ms == -INFINITY ? 0.f : fast_exp2((ms - M) * sl);
        A = fmaf(w, red[s2 * RS + tid], A);
        Lsum = fmaf(w, red[s2 * RS + D + 1], Lsum);
      }
    }
    mine[tid] = A;
    if (tid == 0) {
      mine[D] = M;
      mine[D + 1] = Lsum;
      mine[D + 2] = 0.f;
      mine[D + 3] = 0.f;
    }
  }
  __syncthreads();
  cluster_wait();   // every leader's barrier is set up
  // the head's window branch (leader only; while the other states travel)
  const int hh = bh % p.Hq;
  const bool win = sp == 0 && window_on(p.win, hh);
  float ow = 0.f;
  if (win) ow = window_out<T, D>(p.win, bh, p.Hq, n, sl, reinterpret_cast<float*>(slist));
  const uint32_t leader = cluster_ctarank() - (uint32_t)sp;
  if (sp != 0) {
    // send the state to row sp of the leader's receive rows
    if (tid < RS / 4) {
      const float4 v = reinterpret_cast<const float4*>(mine)[tid];
      st_async_v4(dsmem_map(smem_u32(recv + sp * RS + 4 * tid), leader),
                  make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                             __float_as_uint(v.w)),
                  dsmem_map(smem_u32(bar), leader));
    }
  } else {
    mbar_wait_cluster(bar, 0u, p.err);   // the head's other states are here
  }
  cluster_arrive_relaxed();   // nothing more will arrive here (checked before exit)
  if (sp == 0 && tid < D) {
    // the head's kCombineSplit states, merged in order
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kCombineSplit; ++k) M = fmaxf(M, recv[k * RS + D]);
    float A = 0.f, Lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int k = 0; k < kCombineSplit; ++k) {
        const float ms = recv[k * RS + D];
        const float w = ms == -INFINITY ? 0.f : fast_exp2((ms - M) * sl);
        A = fmaf(w, recv[k * RS + tid], A);
        Lsum = fmaf(w, recv[k * RS + D + 1], Lsum);
      }
    }
    float o = Lsum > 0.f ? A / Lsum : 0.f;
    if (win) o = gate_fuse(o, ow, p.win.gate[bh]);
    store_out<T>(reinterpret_cast<T*>(p.out) + (size_t)bh * D + tid, o);
  }
  cluster_wait();   // no CTA leaves while a state may still be on its way to it
}

}  // namespace lychee
