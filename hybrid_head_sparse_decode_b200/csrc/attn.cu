// attn.cu -- hybrid-head decode attention over one layer (retrieval heads and
// sparse heads in one persistent kernel).
//
// Method: page "LycheeDecode: Accelerating Long-Context LLM Inference via
// Hybrid-Head Sparse Decoding" (paper.rainbus.top/paper/2602.04541), steps (3)
// and (4).  A retrieval head attends to every position j < n_b of its KV group,
// a sparse head only to the positions of its incoming set S.
//
// Work decomposition.  A work item is (sequence b, KV group g, chunk c of
// kChunk positions).  For the G query heads of the group the item needs the
// rows  R = {j in chunk : some head of the group uses j}:  every row when the
// group holds a retrieval head ("dense" group), otherwise the union of the
// heads' sets (read from their membership bitmaps).  Each row of R is read from
// HBM exactly once and serves all G heads (GQA deduplication); each head masks
// the rows that are not its own.
//
// CTA layout (persistent, one CTA per SM, items taken from an atomic counter):
//   * producer warp: builds the item's row list from the bitmaps, then for each
//     tile of TT rows waits for a free ring stage and issues 1-D bulk copies
//     (cp.async.bulk, no tensor map, no multicast) of the K rows and V rows into
//     shared memory, one copy per run of consecutive positions;
//   * NW consumer warps: each owns RW rows of every tile.  q.K: TPR lanes per row,
//     q held in registers (fp32), K widened from bf16 in registers, packed
//     fp32x2 FMA; a reduce-scatter leaves each lane with whole dot products of
//     its heads.  Online softmax state (max m, sum l, accumulator) is kept per
//     warp, so tiles need no CTA-wide barrier.  P.V: one 16-byte chunk of a V
//     row per lane.  At the end of an item the warps' states are merged once
//     and one partial (m, l, acc[d]) per head is written for the combine kernel.
// Tensor cores are not used: per KV row a group does at most 4 * 2d FMAs
// against 2d * sizeof(T) bytes -- a batched GEMV that HBM, not math, bounds.
//
// Logits of retrieval heads (raw q.k in fp32, not divided by sqrt(d)) are
// written to the workspace for the top-k kernel.
#include "common.cuh"
#include "kernels.h"

namespace lychee {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFirst = 1, kLast = 2, kTerm = 4;

template <typename T>
struct Vec16;  // widen one 16-byte chunk to fp32 pairs
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void load(const void* p, float2 (&o)[4]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    o[0] = bf16x2_to_float2(w.x);
    o[1] = bf16x2_to_float2(w.y);
    o[2] = bf16x2_to_float2(w.z);
    o[3] = bf16x2_to_float2(w.w);
  }
};
template <>
struct Vec16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void load(const void* p, float2 (&o)[2]) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    o[0] = make_float2(w.x, w.y);
    o[1] = make_float2(w.z, w.w);
  }
};

// Reduce-scatter of per-lane partial dot products over the TPR lanes of a row.
// cur[0..NCUR) holds one partial per head; each halving level keeps half of the
// heads (upper half when the lane bit M is set) and adds the partner's copy of
// them; once one head is left the remaining levels are plain butterflies.
template <int NCUR, int M>
struct ReduceScatter {
  __device__ __forceinline__ static void run(float* cur, int pp) {
    if constexpr (M >= 1) {
      if constexpr (NCUR > 1) {
        constexpr int HALF = NCUR / 2;
        const bool upper = (pp & M) != 0;
        float keep[HALF];
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const float mine = upper ? cur[HALF + i] : cur[i];
          const float send = upper ? cur[i] : cur[HALF + i];
          keep[i] = mine + __shfl_xor_sync(kFull, send, M);
        }
#pragma unroll
        for (int i = 0; i < HALF; ++i) cur[i] = keep[i];
        ReduceScatter<HALF, M / 2>::run(cur, pp);
      } else {
        cur[0] += __shfl_xor_sync(kFull, cur[0], M);
        ReduceScatter<1, M / 2>::run(cur, pp);
      }
    }
  }
};

template <typename T, int D, int G, int TPR, int NW, int STAGES>
struct AttnCfg {
  static constexpr int E = Vec16<T>::E;           // elements per 16-byte chunk
  static constexpr int CPR = D / E;               // chunks per row
  static constexpr int CPT = CPR / TPR;           // chunks per q.K lane
  static constexpr int RW = 32 / TPR;             // rows per warp per tile
  static constexpr int TT = NW * RW;              // rows per tile
  static constexpr int ROWB = D * (int)sizeof(T); // bytes per K (or V) row
  static constexpr int PVC = CPR;                 // P.V lanes per row
  static constexpr int RGV = 32 / PVC;            // rows a warp covers at once in P.V
  static constexpr int PVR = RW / RGV;            // rows per P.V lane per tile
  static constexpr int GH = G > TPR ? G / TPR : 1;   // heads per q.K lane
  static constexpr int LPH = G < TPR ? TPR / G : 1;  // q.K lanes per head
  static constexpr int NT = (NW + 1) * 32;
  static_assert(CPR % TPR == 0, "TPR must divide the chunks of a row");
  static_assert(PVC <= 32 && RW % RGV == 0, "P.V mapping");
  static_assert(TT <= 64, "run detection uses a 64-bit mask");
  static_assert(kChunk % 32 == 0 && kChunk <= 1024, "producer builds one word per lane");

  // shared memory layout (byte offsets)
  static constexpr size_t kStageKV = (size_t)TT * ROWB;
  static constexpr size_t kQBytes = (size_t)G * D * sizeof(T);
  static constexpr size_t OFF_K = 0;
  static constexpr size_t OFF_V = OFF_K + STAGES * kStageKV;
  static constexpr size_t OFF_Q = OFF_V + STAGES * kStageKV;
  static constexpr size_t OFF_INFO = OFF_Q + STAGES * ((kQBytes + 127) / 128 * 128);
  static constexpr size_t OFF_POS = OFF_INFO + STAGES * 16;
  static constexpr size_t OFF_MASK = OFF_POS + (size_t)STAGES * TT * 4;
  static constexpr size_t OFF_PS = (OFF_MASK + (size_t)STAGES * TT + 15) / 16 * 16;
  static constexpr size_t OFF_MERGE = OFF_PS + (size_t)NW * RW * G * 4;
  static constexpr size_t OFF_LPOS = OFF_MERGE + (size_t)NW * G * (D + 2) * 4;
  static constexpr size_t OFF_LMASK = OFF_LPOS + (size_t)kChunk * 4;
  static constexpr size_t OFF_BAR = (OFF_LMASK + kChunk + 15) / 16 * 16;
  static constexpr size_t SMEM = OFF_BAR + 2 * STAGES * 8;
  static constexpr size_t QSTRIDE = (kQBytes + 127) / 128 * 128;
};

template <typename T, int D, int G, int TPR, int NW, int STAGES>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<T, D, G, TPR, NW, STAGES>;
  constexpr int E = C::E, CPT = C::CPT, RW = C::RW, TT = C::TT, ROWB = C::ROWB;
  constexpr int PVC = C::PVC, RGV = C::RGV, PVR = C::PVR, GH = C::GH, LPH = C::LPH;

  extern __shared__ __align__(128) unsigned char smem[];
  T* Ks = reinterpret_cast<T*>(smem + C::OFF_K);
  T* Vs = reinterpret_cast<T*>(smem + C::OFF_V);
  int4* info = reinterpret_cast<int4*>(smem + C::OFF_INFO);
  int32_t* mpos = reinterpret_cast<int32_t*>(smem + C::OFF_POS);
  uint8_t* mmask = reinterpret_cast<uint8_t*>(smem + C::OFF_MASK);
  float* ps = reinterpret_cast<float*>(smem + C::OFF_PS);
  float* merge = reinterpret_cast<float*>(smem + C::OFF_MERGE);
  int32_t* lpos = reinterpret_cast<int32_t*>(smem + C::OFF_LPOS);
  uint8_t* lmask = reinterpret_cast<uint8_t*>(smem + C::OFF_LMASK);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int Hq = p.Hq, Hkv = p.Hkv, N_max = p.N_max;
  const int nunits = p.B * Hkv;

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_evict_first_policy();
    uint32_t seq = 0;
    bool ok = true;
    for (;;) {
      int item = 0;
      if (lane == 0) item = (int)atomicAdd(p.counter, 1u);
      item = __shfl_sync(kFull, item, 0);
      if (item >= p.n_items) break;
      const int unit = item % nunits, c = item / nunits;
      const int b = unit / Hkv, g = unit % Hkv;
      const int n = min(max(__ldg(&p.seqlens[b]), 1), N_max);
      const int p0 = c * kChunk;
      if (p0 >= n) continue;
      const int p1 = min(p0 + kChunk, n);
      const int h0 = g * G;
      uint32_t rmask = 0;
#pragma unroll
      for (int t = 0; t < G; ++t) rmask |= ((p.role[(h0 + t) >> 5] >> ((h0 + t) & 31)) & 1u) << t;
      const bool dense = rmask != 0;
      // one 32-position word per lane
      const int nwords = (p1 - p0 + 31) >> 5;
      uint32_t bits[G];
      uint32_t uni = 0;
      if (lane < nwords) {
        const int nb = min(32, p1 - p0 - 32 * lane);
        const uint32_t valid = nb == 32 ? kFull : ((1u << nb) - 1u);
        const size_t wbase = (size_t)(b * Hq + h0) * p.nwords + (p0 >> 5) + lane;
#pragma unroll
        for (int t = 0; t < G; ++t) {
          bits[t] = ((rmask >> t) & 1u) ? valid
                                        : (__ldg(&p.bitmaps[wbase + (size_t)t * p.nwords]) & valid);
          uni |= bits[t];
        }
        if (dense) uni = valid;
      } else {
#pragma unroll
        for (int t = 0; t < G; ++t) bits[t] = 0;
      }
      const int cnt = __popc(uni);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      const int total = __shfl_sync(kFull, incl, 31);
      {
        int o = incl - cnt;
        uint32_t u = uni;
        while (u) {
          const int j = __ffs(u) - 1;
          u &= u - 1;
          uint32_t m = 0;
#pragma unroll
          for (int t = 0; t < G; ++t) m |= ((bits[t] >> j) & 1u) << t;
          lpos[o] = p0 + 32 * lane + j;
          lmask[o] = (uint8_t)m;
          ++o;
        }
      }
      __syncwarp();
      if (total == 0) {
        // no row of this chunk is used by any head of the group: empty partials
        if (lane < G) {
          float* ml = p.part_ml + ((size_t)(b * Hq + h0 + lane) * p.nchunk + c) * 2;
          ml[0] = -INFINITY;
          ml[1] = 0.f;
        }
        continue;
      }
      const T* kbase = reinterpret_cast<const T*>(p.k) + (size_t)unit * N_max * D;
      const T* vbase = reinterpret_cast<const T*>(p.v) + (size_t)unit * N_max * D;
      for (int t0 = 0; t0 < total; t0 += TT) {
        const int s = seq % STAGES;
        if (!mbar_wait(&empty[s], ((seq / STAGES) & 1u) ^ 1u, p.err)) {
          ok = false;
          break;
        }
        const int nrows = min(TT, total - t0);
        const int flags = (t0 == 0 ? kFirst : 0) | (t0 + TT >= total ? kLast : 0);
        if (lane == 0) info[s] = make_int4(unit, c, nrows, flags);
        for (int i = lane; i < nrows; i += 32) {
          mpos[s * TT + i] = lpos[t0 + i];
          mmask[s * TT + i] = lmask[t0 + i];
        }
        __syncwarp();
        const uint32_t bytes =
            2u * (uint32_t)nrows * ROWB + ((flags & kFirst) ? (uint32_t)C::kQBytes : 0u);
        if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes);
        __syncwarp();
        T* kd = Ks + (size_t)s * TT * D;
        T* vd = Vs + (size_t)s * TT * D;
        if ((flags & kFirst) && lane == 0) {
          T* qd = reinterpret_cast<T*>(smem + C::OFF_Q + s * C::QSTRIDE);
          bulk_g2s(qd, reinterpret_cast<const T*>(p.q) + (size_t)(b * Hq + h0) * D,
                   (uint32_t)C::kQBytes, &full[s], pol);
        }
        if (dense) {
          if (lane == 0) {
            const size_t off = (size_t)(p0 + t0) * D;
            bulk_g2s(kd, kbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
            bulk_g2s(vd, vbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
          }
        } else {
          // one copy per run of consecutive positions
          uint64_t starts = 0;
#pragma unroll
          for (int half = 0; half < (TT + 31) / 32; ++half) {
            const int i = half * 32 + lane;
            const bool in = i < nrows;
            const int pos = in ? lpos[t0 + i] : 0;
            const int prv = (in && i > 0) ? lpos[t0 + i - 1] : -2;
            const bool st = in && (i == 0 || pos != prv + 1);
            starts |= (uint64_t)__ballot_sync(kFull, st) << (32 * half);
          }
#pragma unroll
          for (int half = 0; half < (TT + 31) / 32; ++half) {
            const int i = half * 32 + lane;
            if (i < nrows && ((starts >> i) & 1ull)) {
              const uint64_t after = (i + 1 < 64) ? (starts >> (i + 1)) << (i + 1) : 0ull;
              const int next = after ? min(__ffsll((long long)after) - 1, nrows) : nrows;
              const int len = next - i;
              const size_t off = (size_t)lpos[t0 + i] * D;
              bulk_g2s(kd + (size_t)i * D, kbase + off, (uint32_t)len * ROWB, &full[s], pol);
              bulk_g2s(vd + (size_t)i * D, vbase + off, (uint32_t)len * ROWB, &full[s], pol);
            }
          }
        }
        ++seq;
      }
      if (!ok) break;
    }
    if (ok) {
      const int s = seq % STAGES;
      if (mbar_wait(&empty[s], ((seq / STAGES) & 1u) ^ 1u, p.err)) {
        if (lane == 0) {
          info[s] = make_int4(0, 0, 0, kTerm);
          mbar_arrive(&full[s]);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int r = lane / TPR, pp = lane % TPR;    // q.K: row within the warp, part
  const int rot = r % CPT;
  const int hb = (G <= TPR) ? pp / LPH : pp * GH;  // first head held after reduce
  const int c16 = lane % PVC, rg = lane / PVC;    // P.V: chunk, row group
  const float sl = p.scale_log2;

  float2 qr[G][CPT][E / 2];
  float m_run[G], l_acc[G];
  float2 acc[G][E / 2];
  float* myps = ps + warp * RW * G;

  uint32_t seq = 0;
  for (;;) {
    const int s = seq % STAGES;
    if (!mbar_wait(&full[s], (seq / STAGES) & 1u, p.err)) return;
    const int4 inf = info[s];
    if (inf.w & kTerm) break;
    const int unit = inf.x, c = inf.y, nrows = inf.z, flags = inf.w;
    const int b = unit / Hkv, h0 = (unit % Hkv) * G;

    if (flags & kFirst) {
      const T* qs = reinterpret_cast<const T*>(smem + C::OFF_Q + s * C::QSTRIDE);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc) {
          const int j = pp + TPR * ((cc + rot) % CPT);
          Vec16<T>::load(qs + h * D + j * E, qr[h][cc]);
        }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_acc[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
      }
    }

    // ---- q.K for row (warp*RW + r), reduce-scatter over the row's TPR lanes
    const int row = warp * RW + r;
    const bool rv = row < nrows;
    float dots[G];
    {
      float2 a2[G];
#pragma unroll
      for (int h = 0; h < G; ++h) a2[h] = make_float2(0.f, 0.f);
      if (rv) {
        const T* krow = Ks + ((size_t)s * TT + row) * D;
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc) {
          const int j = pp + TPR * ((cc + rot) % CPT);
          float2 k2[E / 2];
          Vec16<T>::load(krow + j * E, k2);
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < E / 2; ++e) a2[h] = __ffma2_rn(qr[h][cc][e], k2[e], a2[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) dots[h] = a2[h].x + a2[h].y;
      ReduceScatter<G, TPR / 2>::run(dots, pp);
    }
    const uint32_t rmask = rv ? mmask[s * TT + row] : 0u;
    const int rpos = rv ? mpos[s * TT + row] : 0;
    float sv[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      const int h = hb + i;
      const bool on = (rmask >> h) & 1u;
      const int hq = h0 + h;
      if (on && (pp % LPH) == 0 && ((p.role[hq >> 5] >> (hq & 31)) & 1u))
        p.logits[(size_t)(b * Hq + hq) * N_max + rpos] = dots[i];
      sv[i] = on ? dots[i] : -INFINITY;
    }
    // warp max over rows, then every lane learns the maxima of all G heads
    float mx[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      mx[i] = sv[i];
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1) mx[i] = fmaxf(mx[i], __shfl_xor_sync(kFull, mx[i], o));
    }
    float alpha[G];
    bool rescale = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float t = (G <= TPR) ? __shfl_sync(kFull, mx[0], h * LPH)
                                 : __shfl_sync(kFull, mx[h % GH], h / GH);
      const float mn = fmaxf(m_run[h], t);
      alpha[h] = (mn == m_run[h]) ? 1.f : fast_exp2((m_run[h] - mn) * sl);
      rescale |= (mn != m_run[h]);
      m_run[h] = mn;
    }
    if ((pp % LPH) == 0 && r < RW) {
#pragma unroll
      for (int i = 0; i < GH; ++i) {
        const int h = hb + i;
        float mh = m_run[0];
#pragma unroll
        for (int t = 1; t < G; ++t)
          if (t == h) mh = m_run[t];
        myps[r * G + h] = (sv[i] == -INFINITY) ? 0.f : fast_exp2((sv[i] - mh) * sl);
      }
    }
    __syncwarp();

    // ---- P.V
    if (rescale) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        l_acc[h] *= alpha[h];
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          acc[h][e].x *= alpha[h];
          acc[h][e].y *= alpha[h];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < PVR; ++i) {
      const int rr = rg + RGV * i;
      const int vrow = warp * RW + rr;
      if (vrow < nrows) {
        float pv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pv[h] = myps[rr * G + h];
        float2 v2[E / 2];
        Vec16<T>::load(Vs + ((size_t)s * TT + vrow) * D + c16 * E, v2);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float2 pp2 = make_float2(pv[h], pv[h]);
#pragma unroll
          for (int e = 0; e < E / 2; ++e) acc[h][e] = __ffma2_rn(pp2, v2[e], acc[h][e]);
          l_acc[h] += pv[h];
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    ++seq;

    if (flags & kLast) {
      // ---- merge the warps' states and write one partial per head
#pragma unroll
      for (int o = PVC; o < 32; o <<= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          l_acc[h] += __shfl_xor_sync(kFull, l_acc[h], o);
#pragma unroll
          for (int e = 0; e < E / 2; ++e) {
            acc[h][e].x += __shfl_xor_sync(kFull, acc[h][e].x, o);
            acc[h][e].y += __shfl_xor_sync(kFull, acc[h][e].y, o);
          }
        }
      }
      float* mg = merge + (size_t)warp * G * (D + 2);
      if (rg == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < E / 2; ++e) {
            mg[h * (D + 2) + c16 * E + 2 * e] = acc[h][e].x;
            mg[h * (D + 2) + c16 * E + 2 * e + 1] = acc[h][e].y;
          }
      }
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          mg[h * (D + 2) + D] = m_run[h];
          mg[h * (D + 2) + D + 1] = l_acc[h];
        }
      }
      named_bar_sync(1, NW * 32);
      for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int h = idx / D, dim = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[(w * G + h) * (D + 2) + D]);
        float A = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            const float* e = merge + (w * G + h) * (D + 2);
            const float wt = (e[D] == -INFINITY) ? 0.f : fast_exp2((e[D] - M) * sl);
            A = fmaf(e[dim], wt, A);
            L = fmaf(e[D + 1], wt, L);
          }
        }
        const size_t slot = (size_t)(b * Hq + h0 + h) * p.nchunk + c;
        p.part_acc[slot * D + dim] = A;
        if (dim == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = L;
        }
      }
      named_bar_sync(1, NW * 32);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_acc[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
      }
    }
  }
}

template <typename T, int D, int G, int TPR, int NW, int STAGES>
cudaError_t launch_attn_t(const AttnParams& p, int num_sms, cudaStream_t st) {
  using C = AttnCfg<T, D, G, TPR, NW, STAGES>;
  auto kfn = attn_kernel<T, D, G, TPR, NW, STAGES>;
  static bool attr_set = false;  // per instantiation; set once per process
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = max(1, min(num_sms, p.n_items));
  kfn<<<grid, C::NT, C::SMEM, st>>>(p);
  return cudaGetLastError();
}

// Consumer warps per CTA.  With the producer warp the CTA has NW + 1 warps;
// 8 warps in total puts 2 on each SM sub-partition, which leaves up to 255
// registers per thread for q (held in registers) and the accumulators.
#ifndef LYCHEE_ATTN_NW
#define LYCHEE_ATTN_NW 7
#endif

// Ring depth: about 112-128 KB of K/V tiles in flight per SM, 2..8 stages.
template <typename T, int D, int G, int TPR, int NW>
constexpr int ring_stages() {
  constexpr int bytes = 2 * NW * (32 / TPR) * D * (int)sizeof(T);
  constexpr int s = (128 * 1024) / bytes;
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}

template <typename T, int D, int G, int TPR>
cudaError_t launch_attn_g(const AttnParams& p, int num_sms, cudaStream_t st) {
  constexpr int NW = LYCHEE_ATTN_NW;
  constexpr int STAGES = ring_stages<T, D, G, TPR, NW>();
  static_assert(AttnCfg<T, D, G, TPR, NW, STAGES>::SMEM <= 227 * 1024, "shared memory");
  return launch_attn_t<T, D, G, TPR, NW, STAGES>(p, num_sms, st);
}

template <typename T, int D>
cudaError_t launch_attn_d(const AttnParams& p, int G, int num_sms, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn_g<T, D, 1, 4>(p, num_sms, st);
    case 2: return launch_attn_g<T, D, 2, 4>(p, num_sms, st);
    case 4: return launch_attn_g<T, D, 4, 4>(p, num_sms, st);
    case 8: return launch_attn_g<T, D, 8, 8>(p, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_attn(const AttnParams& p, int dtype, int D, int G, int num_sms,
                        cudaStream_t st) {
  if (dtype == 0) {
    if (D == 128) return launch_attn_d<__nv_bfloat16, 128>(p, G, num_sms, st);
    if (D == 64) return launch_attn_d<__nv_bfloat16, 64>(p, G, num_sms, st);
  } else {
    if (D == 128) return launch_attn_d<float, 128>(p, G, num_sms, st);
    if (D == 64) return launch_attn_d<float, 64>(p, G, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lychee
