// attn.cu -- hybrid-head decode attention over one layer (retrieval heads and
// sparse heads in one persistent kernel).
//
// Method: page "LycheeDecode: Accelerating Long-Context LLM Inference via
// Hybrid-Head Sparse Decoding" (paper.rainbus.top/paper/2602.04541), steps (3)
// and (4).  A retrieval head attends to every position j < n_b of its KV group,
// a sparse head only to the positions of its incoming set S.
//
// Work decomposition.  A work item is (sequence b, chunk c of kChunk positions,
// KV group g); only chunks below n_b exist.  For the G query heads of the group
// the item needs the rows  R = {j in chunk : some head of the group uses j}:
// every row when the group holds a retrieval head ("dense" group), otherwise
// the union of the heads' sets (read from their membership bitmaps).  Each row
// of R is read from HBM once and serves all G heads (GQA deduplication); each
// head masks the rows that are not its own.
//
// CTA layout (persistent, one CTA per SM, items taken from an atomic counter):
//   * NP producer warps: the lead warp claims the next item and loads its
//     bitmap words while the current item streams, and builds the row list;
//     for each tile of TT rows the producers wait for a free ring stage, then a
//     dense tile (consecutive positions) arrives as two 1-D bulk copies
//     (cp.async.bulk, no tensor map, no multicast) of its K rows and V rows,
//     while a sparse tile is gathered row by row with 16-byte cp.async by all
//     producer warps (whole 32-byte sectors, each union row read once);
//   * NW consumer warps: each owns RW rows of every tile.  q.K: TPR lanes per row,
//     q held in registers (fp32), K widened from bf16 in registers, packed
//     fp32x2 FMA; a reduce-scatter leaves each lane with whole dot products of
//     its heads.  The online-softmax state (running max, running sum,
//     accumulator) is kept per warp, so tiles need no CTA-wide barrier, and the
//     accumulator is rescaled only when a running max grows.  P.V: four
//     elements of a V row per lane, probabilities read as pre-duplicated fp32
//     pairs.  At the end of an item the warps' states are merged once and one
//     partial (m, l, acc[d]) per head is written for the combine kernel.
// Tensor cores are not used: per KV row a group does at most 4 * 2d FMAs
// against 2d * sizeof(T) bytes -- a batched GEMV that HBM, not math, bounds.
//
// Logits of retrieval heads (raw q.k in fp32, not divided by sqrt(d)) are
// written to the workspace for the top-k kernel.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace lychee {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFirst = 1, kLast = 2, kTerm = 4, kDense = 8;
constexpr int kMaxBatchCompact = 1024;  // sequences whose chunk counts are kept in smem

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int E = 8;  // elements per 16-byte chunk
  __device__ __forceinline__ static void load16(const void* p, float2 (&o)[4]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    o[0] = bf16x2_to_float2(w.x);
    o[1] = bf16x2_to_float2(w.y);
    o[2] = bf16x2_to_float2(w.z);
    o[3] = bf16x2_to_float2(w.w);
  }
  // four consecutive elements
  __device__ __forceinline__ static void load4(const void* p, float2 (&o)[2]) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    o[0] = bf16x2_to_float2(w.x);
    o[1] = bf16x2_to_float2(w.y);
  }
};
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void load16(const void* p, float2 (&o)[2]) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    o[0] = make_float2(w.x, w.y);
    o[1] = make_float2(w.z, w.w);
  }
  __device__ __forceinline__ static void load4(const void* p, float2 (&o)[2]) {
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

template <typename T, int D, int G, int RQ, int NW, int NP, int STAGES>
struct AttnCfg {
  static constexpr int TPR = 8;                   // q.K lanes per row
  static constexpr int E = Vec<T>::E;             // elements per 16-byte q.K chunk
  static constexpr int CPR = D / E;               // q.K chunks per row
  static constexpr int CPT = CPR / TPR;           // q.K chunks per lane
  static constexpr int RSL = 32 / TPR;            // q.K row slots per warp
  static constexpr int RW = RSL * RQ;             // rows per warp per tile
  static constexpr int TT = NW * RW;              // rows per tile
  static constexpr int ROWB = D * (int)sizeof(T); // bytes per K (or V) row
  static constexpr int PVC = D / 4;               // P.V lanes per row (4 elements each)
  static constexpr int RGV = 32 / PVC;            // rows a warp covers at once in P.V
  static constexpr int PVR = RW / RGV;            // rows per P.V lane per tile
  static constexpr int PVB = 4 * (int)sizeof(T);  // bytes of V per P.V lane and row
  static constexpr int LPH = TPR / G;             // q.K lanes per head
  static constexpr int PPR = ROWB / 16;           // 16-byte pieces per row (gathers)
  static constexpr int RPI = PPR >= 32 ? 1 : 32 / PPR;  // rows per gather instruction
  static constexpr int NT = (NW + NP) * 32;
  static constexpr int MS = D + 4;                // merge row: acc[D], l, m, pad (16-B rows)
  static_assert(CPR % TPR == 0 && CPT >= 1 && (4 % CPT == 0), "q.K mapping");
  static_assert(G <= TPR && TPR % G == 0, "one head per q.K lane");
  static_assert(PVC <= 32 && RW % RGV == 0, "P.V mapping");
  static_assert(TT <= 255, "row count is packed in 8 bits");
  static_assert(kChunk % 32 == 0 && kChunk <= 1024, "producer builds one word per lane");

  // shared memory layout (byte offsets)
  static constexpr int kStageKV = TT * ROWB;
  static constexpr int kQBytes = G * D * (int)sizeof(T);
  static constexpr int QSTRIDE = (kQBytes + 127) / 128 * 128;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * kStageKV;
  static constexpr int OFF_Q = OFF_V + STAGES * kStageKV;
  static constexpr int OFF_INFO = OFF_Q + STAGES * QSTRIDE;
  static constexpr int OFF_POS = OFF_INFO + STAGES * 16;
  static constexpr int OFF_MASK = OFF_POS + STAGES * TT * 4;
  static constexpr int OFF_PS = (OFF_MASK + STAGES * TT + 15) / 16 * 16;
  // per-warp states at an item's end ([NW][G][MS])
  static constexpr int OFF_MERGE = OFF_PS + NW * RW * G * 8;
  static constexpr int OFF_ITEM = OFF_MERGE + NW * G * MS * 4;
  static constexpr int OFF_LPOS = OFF_ITEM + 32;
  static constexpr int OFF_LMASK = OFF_LPOS + kChunk * 4;
  static constexpr int OFF_CUM = (OFF_LMASK + kChunk + 15) / 16 * 16;
  static constexpr int OFF_BAR = (OFF_CUM + (kMaxBatchCompact + 1) * 4 + 15) / 16 * 16;
  static constexpr int SMEM = OFF_BAR + 2 * STAGES * 8;
};

// Item decode shared by the producer: item -> (b, c, g).  With a compact item
// space (B <= kMaxBatchCompact) items enumerate only chunks below n_b, chunk
// major over the concatenated sequences, KV group fastest; cum[b] holds the
// number of chunks of sequences before b.  Otherwise every (b, c < nchunk, g)
// is an item and chunks beyond n_b are skipped by the producer.
__device__ __forceinline__ void decode_item(int item, bool compact, const int* cum, int B,
                                            int Hkv, int nchunk, int& b, int& c, int& g) {
  g = item % Hkv;
  const int cg = item / Hkv;
  if (compact) {
    int lo = 0, hi = B;  // largest b with cum[b] <= cg
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cum[mid] <= cg) lo = mid;
      else hi = mid;
    }
    b = lo;
    c = cg - cum[lo];
  } else {
    b = cg / nchunk;
    c = cg % nchunk;
  }
}

template <typename T, int D, int G, int RQ, int NW, int NP, int STAGES>
__device__ __forceinline__ void consumer_loop(const AttnParams& p, unsigned char* smem,
                                              uint64_t* full, uint64_t* empty);

template <typename T, int D, int G, int RQ, int NW, int NP, int STAGES>
__global__ void __launch_bounds__((NW + NP) * 32, 1)
    attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<T, D, G, RQ, NW, NP, STAGES>;
  constexpr int TPR = C::TPR, E = C::E, CPT = C::CPT, RSL = C::RSL, RW = C::RW, TT = C::TT;
  constexpr int ROWB = C::ROWB, PVC = C::PVC, RGV = C::RGV, PVR = C::PVR, PVB = C::PVB;
  constexpr int LPH = C::LPH, PPR = C::PPR, RPI = C::RPI, MS = C::MS;

  extern __shared__ __align__(128) unsigned char smem[];
  int4* info = reinterpret_cast<int4*>(smem + C::OFF_INFO);
  int32_t* mpos = reinterpret_cast<int32_t*>(smem + C::OFF_POS);
  uint8_t* mmask = reinterpret_cast<uint8_t*>(smem + C::OFF_MASK);
  float* merge = reinterpret_cast<float*>(smem + C::OFF_MERGE);
  int* item_desc = reinterpret_cast<int*>(smem + C::OFF_ITEM);
  int32_t* lpos = reinterpret_cast<int32_t*>(smem + C::OFF_LPOS);
  uint8_t* lmask = reinterpret_cast<uint8_t*>(smem + C::OFF_LMASK);
  int* cum = reinterpret_cast<int*>(smem + C::OFF_CUM);
  // per stage: full (row list, q and K/V rows landed; one arrival per producer
  // warp), empty (every consumer warp is done with the stage)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = p.Hq, Hkv = p.Hkv, N_max = p.N_max, B = p.B;
  const bool compact = B <= kMaxBatchCompact;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], NP);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  if (warp == NW && compact) {
    // chunk counts per sequence -> exclusive prefix in cum[0..B]
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int n = b < B ? min(max(__ldg(&p.seqlens[b]), 1), N_max) : 0;
      const int nc = (n + kChunk - 1) / kChunk;
      int incl = nc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < B) cum[b] = carry + incl - nc;
      carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) cum[B] = carry;
  }
  __syncthreads();

  if (warp >= NW) {
    // ------------------------------------------------------- producer group
    const int pw = warp - NW;              // 0 leads: claims, row lists, TMA
    const int n_items = compact ? cum[B] * Hkv : p.n_items;
    const uint64_t pol = l2_evict_first_policy();
    uint32_t s = 0, ph = 0;                // ring stage and its phase parity
    bool ok = true;

    // lead only: claim an item (lane 0) and load what building its row list needs
    auto claim = [&]() -> int { return lane == 0 ? (int)atomicAdd(p.counter, 1u) : 0; };
    auto prefetch = [&](int item, int& nraw, uint32_t (&w)[G]) {
      nraw = 1;
#pragma unroll
      for (int t = 0; t < G; ++t) w[t] = 0u;
      if (item >= n_items) return;
      int b, c, g;
      decode_item(item, compact, cum, B, Hkv, p.nchunk, b, c, g);
      nraw = __ldg(&p.seqlens[b]);
      const int word = c * (kChunk / 32) + lane;
      if (lane < kChunk / 32 && word < p.nwords) {
        const size_t wbase = (size_t)(b * Hq + g * G) * p.nwords + word;
#pragma unroll
        for (int t = 0; t < G; ++t) w[t] = __ldg(&p.bitmaps[wbase + (size_t)t * p.nwords]);
      }
    };
    if (pw == 0 && blockIdx.x == 0) {
      for (int bb = lane; bb < B; bb += 32) {
        const int n_raw = __ldg(&p.seqlens[bb]);
        if (n_raw < 1 || n_raw > N_max) flag_error(p.err, kErrBadSeqlen);
        if (p.k_per_seq && __ldg(&p.k_per_seq[bb]) < 1) flag_error(p.err, kErrBadBudget);
      }
    }
    int cur = 0, cur_n = 1, claimed = 0;
    uint32_t cur_w[G];
    if (pw == 0) {
      cur = __shfl_sync(kFull, claim(), 0);
      prefetch(cur, cur_n, cur_w);
      claimed = claim();
    }

    for (;;) {
      // -- the lead builds the next item's row list; the group then streams it
      int total = 0, b = 0, c = 0, g = 0, p0 = 0;
      bool dense = false;
      if (pw == 0) {
        int nxt_n = 1, nxt = 0;
        uint32_t nxt_w[G];
        for (;;) {   // skip items without rows
          if (cur >= n_items) {
            total = -1;
            break;
          }
          decode_item(cur, compact, cum, B, Hkv, p.nchunk, b, c, g);
          const int n = min(max(cur_n, 1), N_max);
          p0 = c * kChunk;
          const int h0 = g * G;
          // claim and load the item after this one while this one streams
          nxt = __shfl_sync(kFull, claimed, 0);
          prefetch(nxt, nxt_n, nxt_w);
          claimed = claim();
          if (p0 < n) {
            const int p1 = min(p0 + kChunk, n);
            uint32_t rmask = 0;
#pragma unroll
            for (int t = 0; t < G; ++t)
              rmask |= ((p.role[(h0 + t) >> 5] >> ((h0 + t) & 31)) & 1u) << t;
            dense = rmask != 0;
            const int nwords = (p1 - p0 + 31) >> 5;
            uint32_t bits[G];
            uint32_t uni = 0;
            const int nb = lane < nwords ? min(32, p1 - p0 - 32 * lane) : 0;
            const uint32_t valid = nb >= 32 ? kFull : ((1u << nb) - 1u);
#pragma unroll
            for (int t = 0; t < G; ++t) {
              bits[t] = ((rmask >> t) & 1u) ? valid : (cur_w[t] & valid);
              uni |= bits[t];
            }
            if (dense) uni = valid;
            const int cnt = __popc(uni);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(kFull, incl, o);
              if (lane >= o) incl += y;
            }
            total = __shfl_sync(kFull, incl, 31);
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
          cur = nxt;
          cur_n = nxt_n;
#pragma unroll
          for (int t = 0; t < G; ++t) cur_w[t] = nxt_w[t];
          if (p0 < n) break;   // chunks beyond n_b exist only without the compact space
        }
        if (lane == 0) {
          item_desc[0] = total;
          item_desc[1] = b;
          item_desc[2] = c;
          item_desc[3] = g;
          item_desc[4] = p0;
          item_desc[5] = dense ? 1 : 0;
        }
      }
      named_bar_sync(2, NP * 32);            // row list and descriptor ready
      total = item_desc[0];
      b = item_desc[1];
      c = item_desc[2];
      g = item_desc[3];
      p0 = item_desc[4];
      dense = item_desc[5] != 0;
      const int h0 = g * G;
      const int unit = b * Hkv + g;
      const T* kbase = reinterpret_cast<const T*>(p.k) + (size_t)unit * N_max * D;
      const T* vbase = reinterpret_cast<const T*>(p.v) + (size_t)unit * N_max * D;
      // the end is one entry; a chunk no head of the group uses is one empty tile
      const int ntile = total <= 0 ? 1 : (total + TT - 1) / TT;
      for (int tt = 0; tt < ntile; ++tt) {
        const int t0 = tt * TT;
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err)) {
          ok = false;
          break;
        }
        const int nrows = total < 0 ? 0 : min(TT, total - t0);
        const int flags = total < 0 ? kTerm
                                    : ((t0 == 0 ? kFirst : 0) | (t0 + TT >= total ? kLast : 0) |
                                       (dense ? kDense : 0));
        T* kd = reinterpret_cast<T*>(smem + C::OFF_K + s * C::kStageKV);
        T* vd = reinterpret_cast<T*>(smem + C::OFF_V + s * C::kStageKV);
        if (pw == 0) {
          if (lane == 0) info[s] = make_int4(b, h0, (c << 8) | nrows, flags);
          for (int i = lane; i < nrows; i += 32) {
            mpos[s * TT + i] = lpos[t0 + i];
            mmask[s * TT + i] = lmask[t0 + i];
          }
        }
        if (!(flags & (kDense | kTerm))) {
          // gather the listed rows with 16-byte copies, split over the group;
          // each lane's copies are tracked by the stage's full barrier
          for (int r0 = pw * RPI; r0 < nrows; r0 += NP * RPI) {
#pragma unroll
            for (int pc2 = 0; pc2 < (PPR + 31) / 32; ++pc2) {
              const int row = r0 + (PPR >= 32 ? 0 : lane / PPR);
              const int piece = PPR >= 32 ? pc2 * 32 + lane : lane % PPR;
              if (row < nrows && piece < PPR) {
                const size_t src = (size_t)lpos[t0 + row] * D + piece * E;
                const int dst = row * D + piece * E;
                cp_async16(kd + dst, kbase + src);
                cp_async16(vd + dst, vbase + src);
              }
            }
          }
          cp_async_mbar_arrive(&full[s]);
        }
        __syncwarp();
        if (lane == 0) {
          if (pw == 0) {
            const uint32_t bytes = ((flags & kDense) ? 2u * (uint32_t)nrows * ROWB : 0u) +
                                   ((flags & kFirst) ? (uint32_t)C::kQBytes : 0u);
            fence_proxy_async_smem();
            if (bytes) mbar_arrive_expect_tx(&full[s], bytes);
            else mbar_arrive(&full[s]);
            if (flags & kFirst) {
              T* qd = reinterpret_cast<T*>(smem + C::OFF_Q + s * C::QSTRIDE);
              bulk_g2s(qd, reinterpret_cast<const T*>(p.q) + (size_t)(b * Hq + h0) * D,
                       (uint32_t)C::kQBytes, &full[s], pol);
            }
            if (flags & kDense) {
              const size_t off = (size_t)(p0 + t0) * D;
              bulk_g2s(kd, kbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
              bulk_g2s(vd, vbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
            }
          } else {
            mbar_arrive(&full[s]);
          }
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok || total < 0) break;
      named_bar_sync(2, NP * 32);            // every gather of this item was issued
    }
  } else {
    consumer_loop<T, D, G, RQ, NW, NP, STAGES>(p, smem, full, empty);
  }
  // ---- the last CTA to leave resets the launch counters for the next launch
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.exits, 1u) == gridDim.x - 1) {
      *p.counter = 0u;
      *p.exits = 0u;
      __threadfence();
    }
  }
}

// Consumer warps of attn_kernel (see the file comment).
template <typename T, int D, int G, int RQ, int NW, int NP, int STAGES>
__device__ __forceinline__ void consumer_loop(const AttnParams& p, unsigned char* smem,
                                              uint64_t* full, uint64_t* empty) {
  using C = AttnCfg<T, D, G, RQ, NW, NP, STAGES>;
  constexpr int TPR = C::TPR, E = C::E, CPT = C::CPT, RSL = C::RSL, RW = C::RW, TT = C::TT;
  constexpr int ROWB = C::ROWB, PVC = C::PVC, RGV = C::RGV, PVR = C::PVR, PVB = C::PVB;
  constexpr int LPH = C::LPH, MS = C::MS;
  const int4* info = reinterpret_cast<const int4*>(smem + C::OFF_INFO);
  const int32_t* mpos = reinterpret_cast<const int32_t*>(smem + C::OFF_POS);
  const uint8_t* mmask = reinterpret_cast<const uint8_t*>(smem + C::OFF_MASK);
  float* merge = reinterpret_cast<float*>(smem + C::OFF_MERGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = p.Hq, N_max = p.N_max;

  const int r = lane / TPR, pp = lane % TPR;     // q.K: row slot, part
  const int rot = r % CPT;                       // same for every row of the lane
  const int hb = pp / LPH;                       // the head this lane reduces to
  const bool writer = (pp % LPH) == 0;           // one lane per (row, head) writes
  const int pc = lane % PVC, rg = lane / PVC;    // P.V: 4-element chunk, row group
  const float sl = p.scale_log2;

  // lane-constant shared-memory byte offsets (stage 0)
  int koff[CPT];
#pragma unroll
  for (int cc = 0; cc < CPT; ++cc)
    koff[cc] = C::OFF_K + (warp * RW + r) * ROWB + (pp + TPR * ((cc + rot) % CPT)) * 16;
  const int voff = C::OFF_V + (warp * RW + rg) * ROWB + pc * PVB;
  const int pw_off = C::OFF_PS + ((warp * RW + r) * G + hb) * 8;   // p writes (slot r)
  const int pr_off = C::OFF_PS + (warp * RW + rg) * G * 8;         // p reads (row rg)
  const int row0 = warp * RW + r;                                  // first q.K row

  float2 qr[G][CPT][E / 2];
  float m_run[G];
  float m_own = -INFINITY, msl = 0.f, l_own = 0.f;
  float2 acc[G][2];
  float* lg = nullptr;        // logits row of the lane's head (retrieval heads only)
  bool lg_on = false;
  int b = 0, h0 = 0, c = 0;

  uint32_t s = 0, ph = 0;
  for (;;) {
    if (!mbar_wait(&full[s], ph, p.err)) break;
    const int4 inf = info[s];
    if (inf.w & kTerm) break;
    const int nrows = inf.z & 255, flags = inf.w;
    const int kst = s * C::kStageKV;           // stage offset in the K and V rings

    if (flags & kFirst) {
      b = inf.x;
      h0 = inf.y;
      c = inf.z >> 8;
      const int hq = h0 + hb;
      lg_on = writer && ((p.role[hq >> 5] >> (hq & 31)) & 1u);
      lg = p.logits + (size_t)(b * Hq + hq) * N_max;
      const T* qs = reinterpret_cast<const T*>(smem + C::OFF_Q + s * C::QSTRIDE);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc) {
          const int j = pp + TPR * ((cc + rot) % CPT);
          Vec<T>::load16(qs + h * D + j * E, qr[h][cc]);
        }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        acc[h][0] = acc[h][1] = make_float2(0.f, 0.f);
      }
      m_own = -INFINITY;
      msl = 0.f;
      l_own = 0.f;
    }

    // one tile; WHOLE: every row of the tile exists (no per-row tests)
    auto tile = [&](auto whole_tag) {
      constexpr bool WHOLE = decltype(whole_tag)::value;
      // ---- q.K for the lane's RQ rows
      float sv[RQ];
      const int mrow = s * TT + row0;
#pragma unroll
      for (int i = 0; i < RQ; ++i) {
        const bool rv = WHOLE || (row0 + RSL * i) < nrows;
        float2 a2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) a2[h] = make_float2(0.f, 0.f);
        if (rv) {
#pragma unroll
          for (int cc = 0; cc < CPT; ++cc) {
            float2 k2[E / 2];
            Vec<T>::load16(smem + kst + koff[cc] + i * RSL * ROWB, k2);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < E / 2; ++e) a2[h] = __ffma2_rn(qr[h][cc][e], k2[e], a2[h]);
          }
        }
        float dots[G];
#pragma unroll
        for (int h = 0; h < G; ++h) dots[h] = a2[h].x + a2[h].y;
        ReduceScatter<G, TPR / 2>::run(dots, pp);
        const uint32_t rmask = rv ? (uint32_t)mmask[mrow + RSL * i] : 0u;
        const bool on = (rmask >> hb) & 1u;
        if (on && lg_on) lg[mpos[mrow + RSL * i]] = dots[0];
        sv[i] = on ? dots[0] : -INFINITY;
      }
      // ---- running maximum of every head over the warp's rows
      float mx = sv[0];
#pragma unroll
      for (int i = 1; i < RQ; ++i) mx = fmaxf(mx, sv[i]);
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
      float tmax[G];
      bool grow = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        tmax[h] = __shfl_sync(kFull, mx, h * LPH);
        grow |= tmax[h] > m_run[h];
      }
      if (grow) {  // warp-uniform: every lane holds the same maxima
        float a_own = 1.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mn = fmaxf(m_run[h], tmax[h]);
          const float al = (mn == m_run[h]) ? 1.f : fast_exp2((m_run[h] - mn) * sl);
          m_run[h] = mn;
          const float2 a2 = make_float2(al, al);
          acc[h][0] = __fmul2_rn(acc[h][0], a2);
          acc[h][1] = __fmul2_rn(acc[h][1], a2);
          if (h == hb) {
            m_own = mn;
            a_own = al;
          }
        }
        l_own *= a_own;
        msl = (m_own == -INFINITY) ? 0.f : m_own * sl;
      }
      // ---- probabilities of the lane's rows, shared as (p, p) pairs
#pragma unroll
      for (int i = 0; i < RQ; ++i) {
        const float pr = fast_exp2(fmaf(sv[i], sl, -msl));
        l_own += pr;
        if (writer)
          *reinterpret_cast<float2*>(smem + pw_off + i * RSL * G * 8) = make_float2(pr, pr);
      }
      __syncwarp();
      // ---- P.V: lane (pc, rg) accumulates elements [4pc, 4pc+4) of rows rg + RGV*i
#pragma unroll
      for (int i = 0; i < PVR; ++i) {
        if (WHOLE || (warp * RW + rg + RGV * i) < nrows) {
          const unsigned char* pb = smem + pr_off + i * RGV * G * 8;
          float2 pr2[G];
          if constexpr (G == 1) {
            pr2[0] = *reinterpret_cast<const float2*>(pb);
          } else {
#pragma unroll
            for (int h = 0; h < G; h += 2) {
              const float4 t = *reinterpret_cast<const float4*>(pb + h * 8);
              pr2[h] = make_float2(t.x, t.y);
              pr2[h + 1] = make_float2(t.z, t.w);
            }
          }
          float2 v2[2];
          Vec<T>::load4(smem + kst + voff + i * RGV * ROWB, v2);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            acc[h][0] = __ffma2_rn(pr2[h], v2[0], acc[h][0]);
            acc[h][1] = __ffma2_rn(pr2[h], v2[1], acc[h][1]);
          }
        }
      }
    };
    if (nrows == TT) tile(std::true_type{});
    else tile(std::false_type{});
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == STAGES) {
      s = 0;
      ph ^= 1u;
    }

    if (flags & kLast) {
      // ---- merge the warps' states in a fixed order and write one partial per head
      float l_w = l_own;
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1) l_w += __shfl_xor_sync(kFull, l_w, o);
#pragma unroll
      for (int o = PVC; o < 32; o <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            acc[h][e].x += __shfl_xor_sync(kFull, acc[h][e].x, o);
            acc[h][e].y += __shfl_xor_sync(kFull, acc[h][e].y, o);
          }
      float* mg = merge + warp * G * MS;
      if (rg == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h)
          *reinterpret_cast<float4*>(mg + h * MS + pc * 4) =
              make_float4(acc[h][0].x, acc[h][0].y, acc[h][1].x, acc[h][1].y);
      }
      if (r == 0 && writer) {
        mg[hb * MS + D] = l_w;
        mg[hb * MS + D + 1] = m_own;
      }
      named_bar_sync(1, NW * 32);
      for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int h = idx / D, dim = idx % D;
        float M = -INFINITY;
#pragma unroll 4
        for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[(w * G + h) * MS + D + 1]);
        float A = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll 4
          for (int w = 0; w < NW; ++w) {
            const float* e = merge + (w * G + h) * MS;
            const float wt = (e[D + 1] == -INFINITY) ? 0.f : fast_exp2((e[D + 1] - M) * sl);
            A = fmaf(e[dim], wt, A);
            L = fmaf(e[D], wt, L);
          }
        }
        const size_t slot = (size_t)(b * Hq + h0 + h) * p.nchunk + c;
        p.part_acc[slot * D + dim] = A;
        if (dim == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = L;
        }
      }
      named_bar_sync(1, NW * 32);   // the slots are rewritten at the next item's end
    }
  }
}

template <typename T, int D, int G, int RQ, int NW, int NP, int STAGES>
cudaError_t launch_attn_t(const AttnParams& p, int num_sms, cudaStream_t st) {
  using C = AttnCfg<T, D, G, RQ, NW, NP, STAGES>;
  auto kfn = attn_kernel<T, D, G, RQ, NW, NP, STAGES>;
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

// 16 warps per CTA: NW consumers and NP producers, 4 warps on each SM
// sub-partition with up to 128 registers per thread.  q.K uses 8 lanes per row
// (64 q values in registers for G <= 4) and RQ rows per lane; the producers
// gather sparse rows with 16-byte copies and stream dense rows with TMA.
// G = 8 keeps 128 q values per lane and runs 8 warps (up to 255 registers).
#ifndef LYCHEE_ATTN_NW
#define LYCHEE_ATTN_NW 12
#endif
#ifndef LYCHEE_ATTN_NP
#define LYCHEE_ATTN_NP 4
#endif
#ifndef LYCHEE_ATTN_RING_KB
#define LYCHEE_ATTN_RING_KB 150
#endif

// Ring depth: about LYCHEE_ATTN_RING_KB of K/V tiles per SM, 2..8 stages.
template <typename T, int D, int G, int RQ, int NW>
constexpr int ring_stages() {
  constexpr int bytes = 2 * NW * 4 * RQ * D * (int)sizeof(T) +
                        (G * D * (int)sizeof(T) + 127) / 128 * 128;   // K, V tiles and q
  constexpr int s = (LYCHEE_ATTN_RING_KB * 1024) / bytes;
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}

template <typename T, int D, int G, int RQ, int NW, int NP>
cudaError_t launch_attn_g(const AttnParams& p, int num_sms, cudaStream_t st) {
  constexpr int STAGES = ring_stages<T, D, G, RQ, NW>();
  static_assert(AttnCfg<T, D, G, RQ, NW, NP, STAGES>::SMEM <= 227 * 1024, "shared memory");
  return launch_attn_t<T, D, G, RQ, NW, NP, STAGES>(p, num_sms, st);
}

template <typename T, int D>
cudaError_t launch_attn_d(const AttnParams& p, int G, int num_sms, cudaStream_t st) {
  constexpr int NW = LYCHEE_ATTN_NW, NP = LYCHEE_ATTN_NP;
  constexpr int RQ = (sizeof(T) * D > 256) ? 1 : 2;   // fp32 rows of 512 bytes: one per lane
  switch (G) {
    case 1: return launch_attn_g<T, D, 1, RQ, NW, NP>(p, num_sms, st);
    case 2: return launch_attn_g<T, D, 2, RQ, NW, NP>(p, num_sms, st);
    case 4: return launch_attn_g<T, D, 4, RQ, NW, NP>(p, num_sms, st);
    case 8: return launch_attn_g<T, D, 8, 1, 6, 2>(p, num_sms, st);
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
