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
// of R is read from HBM once into shared memory and serves every head of the
// group that uses it (GQA deduplication).
//
// CTA layout (persistent, one CTA per SM, items taken from an atomic counter):
//   * a builder warp claims items and turns each into its row list R and
//     what the consumers need to know which head uses which row: for the
//     tensor-core consumers each head's membership words of the chunk, for
//     the fp32 consumers each sparse head's list of the rows of R it uses
//     (with per-tile offsets) and a share of the consumer warps for every head
//     proportional to its rows.  It fills two alternating item buffers, so the
//     next item is built while the current one streams and is consumed.
//   * streaming warps move each built item through a ring of shared-memory
//     stages in tiles of TT rows of R.
//     - bf16 caches: a stage holds K and V as planes of 128-byte half rows
//       (64 dimensions each) with a 128-byte swizzle.  A dense tile
//       (consecutive positions) arrives as TMA tiled loads, one box per plane
//       of K and of V, issued by the first streaming warp; a sparse tile is
//       gathered row by row by 16-byte cp.async spread over every streaming
//       warp, each piece written to its swizzled slot.
//     - fp32 caches: a stage holds the rows as they are in HBM.  A dense tile
//       arrives as two 1-D bulk copies (cp.async.bulk); a sparse tile over
//       two paths at once, part of the rows as TMA tile::gather4 copies (four
//       rows each, through a tensor map over the cache rows) issued by the
//       first streaming warp, the rest as 16-byte cp.async by the others.
//     Whole 32-byte sectors either way; no copy uses multicast.
//   * NW consumer warps, in one of two forms.
//     - bf16 caches (consumer_loop_mma): a warp takes whole slabs of 16 rows
//       and serves every head of the group on them at once on the tensor cores
//       (mma.sync m16n8k16, bf16 operands, fp32 accumulation): S^T = K q^T for
//       the slab, scores of rows a head does not use set to -inf from the
//       heads' membership words, an online softmax per head with a lazy
//       maximum, O^T += V^T P with P rounded to bf16; the fragments of K and
//       of V^T come straight from the swizzled planes by ldmatrix (transposing
//       for V).  A row of the union costs the same few instructions whichever
//       heads use it, so the warps
//       keep pace with HBM; the arithmetic is a skinny GEMM (at most 8 heads
//       wide) that the warp-level MMA serves without any staging.
//     - fp32 caches (consumer_loop): during an item each warp serves one head
//       and only that head's rows (pairs (row, head)).  Four lanes share a
//       pair, each holding a quarter of q (fp32 registers) and of the output
//       accumulator; eight pairs are in flight per warp.  q.K with packed
//       fp32x2 FMA and two shuffles to finish the dot product, the same lazy
//       online softmax per pair slot, P.V on the same lanes and rows.
//     At the end of an item the fp32 consumers write each warp's partial state
//     (m, l, acc[d]) for each head it served to its own slot of the workspace;
//     the tensor-core consumers first merge their warps' states of each head
//     in shared memory (a fixed order) and write one.  The combine merges the
//     states and chunks in a fixed order, so the result does not depend on
//     scheduling.
// Logits of retrieval heads (raw q.k in fp32, not divided by sqrt(d)) are
// written to the workspace for the top-k kernel.
#include <type_traits>

#include "combine_body.cuh"
#include "common.cuh"
#include "kernels.h"

namespace lychee {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFirst = 1, kLast = 2, kTerm = 4, kDense = 8;
constexpr int kMaxBatchCompact = 1024;  // sequences whose chunk counts are kept in smem
constexpr int kLanesPerPair = 4;        // lanes sharing one (row, head) pair
constexpr int kPairsPerBatch = 32 / kLanesPerPair;
constexpr float kLazyLog2 = 8.f;        // rescale when a probability would exceed 2^8
constexpr uint8_t kNoHead = 0xff;

#ifndef LYCHEE_ATTN_ILP
#define LYCHEE_ATTN_ILP 2   // batches of pairs a consumer warp works on at once
#endif
// Batches in flight per consumer warp for element type T and head dim D: rows
// of 512 bytes (fp32, d = 128) keep one (twice the registers per chunk).
template <typename T, int D>
constexpr int ilp_of() {
  return D * (int)sizeof(T) > 256 ? 1 : LYCHEE_ATTN_ILP;
}

// Register split between the warpgroups of the fp32-FMA kernel (setmaxnreg):
// the producer warpgroup gives registers back, the consumer warpgroups take
// them.  The block launches with 65536 / threads registers per thread (checked
// on the host before the launch); the split must fit in them.
#ifndef LYCHEE_ATTN_REGSPLIT
#define LYCHEE_ATTN_REGSPLIT 1
#endif
#ifndef LYCHEE_ATTN_PROD_REGS
#define LYCHEE_ATTN_PROD_REGS 80
#endif
#ifndef LYCHEE_ATTN_CONS_REGS
#define LYCHEE_ATTN_CONS_REGS 136
#endif
constexpr int kProdRegs = LYCHEE_ATTN_PROD_REGS;
constexpr int kConsRegs = LYCHEE_ATTN_CONS_REGS;

// fp32 caches: sparse tiles take two copy paths at once, the first
// LYCHEE_ATTN_TMA_ROWS/16 of a tile's rows as TMA tile::gather4 copies issued by
// the first streaming warp, the rest as 16-byte cp.async by the other streaming
// warps.  0: cp.async only (always so with bf16 caches, whose V rows land in
// the swizzled layout).
#ifndef LYCHEE_ATTN_TMA_ROWS
#define LYCHEE_ATTN_TMA_ROWS 8
#endif
// bf16 caches: consumer warps contract on the tensor cores (mma.sync, see
// consumer_loop_mma); 0: the fp32-FMA consumer for every type.
#ifndef LYCHEE_ATTN_MMA
#define LYCHEE_ATTN_MMA 1
#endif
template <typename T>
constexpr bool mma_path() {
  return LYCHEE_ATTN_MMA && std::is_same<T, __nv_bfloat16>::value;
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int E = 8;  // elements per 16-byte chunk
  __device__ __forceinline__ static void widen(uint4 w, float2 (&o)[4]) {
    o[0] = bf16x2_to_float2(w.x);
    o[1] = bf16x2_to_float2(w.y);
    o[2] = bf16x2_to_float2(w.z);
    o[3] = bf16x2_to_float2(w.w);
  }
  __device__ __forceinline__ static void load16(const void* p, float2 (&o)[4]) {
    widen(*reinterpret_cast<const uint4*>(p), o);
  }
};
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void widen(uint4 w, float2 (&o)[2]) {
    o[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
    o[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
  }
  __device__ __forceinline__ static void load16(const void* p, float2 (&o)[2]) {
    widen(*reinterpret_cast<const uint4*>(p), o);
  }
};

template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
struct AttnCfg {
  static constexpr int E = Vec<T>::E;             // elements per 16-byte chunk
  static constexpr int DL = D / kLanesPerPair;    // dimensions per lane
  static constexpr int CPL = DL / E;              // 16-byte chunks per lane
  static constexpr int ROWB = D * (int)sizeof(T); // bytes per K (or V) row
  static constexpr int PPR = ROWB / 16;           // 16-byte pieces per row (gathers)
  static constexpr int RPI = PPR >= 32 ? 1 : 32 / PPR;  // rows per gather instruction
  static constexpr int NT = (NW + NP) * 32;
  // register split (setmaxnreg, fp32-FMA consumers): the block launches with
  // LREGS registers per thread, the producer warpgroups drop to PREGS, the
  // consumer ones rise to CREGS
  static constexpr bool RSPLIT = !mma_path<T>() && ilp_of<T, D>() > 1 && LYCHEE_ATTN_REGSPLIT;
  static constexpr int LREGS = (65536 / NT) & ~7;
  static constexpr int PREGS = kProdRegs;
  static constexpr int CREGS = kConsRegs;
  static_assert(!RSPLIT || (NW % 4 == 0 && NP % 4 == 0 && NP * 32 * PREGS + NW * 32 * CREGS <= NT * LREGS),
                "register split: whole warpgroups, within the launch's registers");
  static constexpr int NS = NP - 1;               // streaming warps (all producers but the builder)
  static constexpr int MAXT = (kChunk + TT - 1) / TT;   // tiles per item at most
  static_assert(CPL >= 2 && DL % E == 0 && CPL % 2 == 0, "lane mapping");
  static_assert(TT % kPairsPerBatch == 0 && TT % 4 == 0 && TT <= 255, "tile rows");
  static constexpr bool MMA = mma_path<T>();
  // tensor-core consumers: K and V tiles in swizzled planes (below), sparse
  // rows by 16-byte copies only
  static constexpr bool SWZ = MMA;
  static constexpr int TMA_ROWS = MMA ? 0 : LYCHEE_ATTN_TMA_ROWS;
  static constexpr int NPL = ROWB / 128;          // planes (SWZ): 64 dimensions each
  static constexpr int PLANE = TT * 128;          // bytes per plane of a stage's K or V
  static_assert(!SWZ || (ROWB % 128 == 0 && TT % 16 == 0),
                "swizzled planes: whole 128-byte half rows, 16-row boxes");
  static constexpr int ALIGN = SWZ ? 1024 : 128;  // the 128-byte swizzle repeats every 1024 bytes
  static_assert(MMA ? (G <= 8 && NW <= kPartSlots && TT % 16 == 0)
                    : (G <= NW && NW <= kPartSlots && NW <= 16),
                "warps per head fit the partial slots; tensor-core slabs of 16 rows");
  static_assert(NP >= 2, "a builder and at least one streaming warp");
  static_assert(kChunk % 32 == 0 && kChunk <= 1024, "builder holds one word per lane");
  static_assert(MAXT < 32, "one lane per tile start");

  // item buffer (two of them): descriptor, then for the fp32-FMA consumers the
  // warp assignment, where each tile starts in each sparse head's row list and
  // the row lists (union indices of the head's rows, in order), for the
  // tensor-core consumers each head's membership word for every 32 positions
  // of the chunk ([word][8] u32, head t at t; heads >= G zero), then the gather
  // positions
  static constexpr int ASGB = NW + G;             // warp -> (head, slot), warps per head
  static constexpr int IB_ASG = 32;
  static constexpr int IB_TST = IB_ASG + (MMA ? 0 : (ASGB + 15) / 16 * 16);   // [G][32] u16
  static constexpr int IB_HROW = IB_TST + (MMA ? 0 : G * 32 * 2);             // [G][kChunk] u16
  static constexpr int IB_HW = IB_HROW + (MMA ? 0 : G * kChunk * 2);          // [kChunk/32][8] u32
  static constexpr int IB_LPOS = IB_HW + (MMA ? kChunk : 0);                  // [kChunk] i32
  static_assert(IB_LPOS % 16 == 0, "positions read four at a time");
  static constexpr int IBUF = IB_LPOS + kChunk * 4;

  // shared memory layout (byte offsets from an ALIGN-byte aligned base)
  static constexpr int kStageKV = TT * ROWB;
  static constexpr int kQBytes = G * D * (int)sizeof(T);
  static constexpr int QSTRIDE = (kQBytes + 127) / 128 * 128;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * kStageKV;
  static constexpr int OFF_Q = OFF_V + STAGES * kStageKV;
  static constexpr int OFF_INFO = OFF_Q + STAGES * QSTRIDE;             // [STAGES][2] int4
  static constexpr int OFF_ITEM = OFF_INFO + STAGES * 32;               // [2][IBUF]
  static constexpr int OFF_CUM = OFF_ITEM + 2 * IBUF;
  // tensor-core consumers: the warps' states of an item's heads, merged into
  // one per head before they go out ([NW][MRGH][D + 2] fp32, up to four heads
  // a round)
  static constexpr int MRGH = G < 4 ? G : 4;
  static constexpr int OFF_MRG = (OFF_CUM + (kMaxBatchCompact + 1) * 4 + 15) / 16 * 16;
  static constexpr int MRGB = MMA ? NW * MRGH * (D + 2) * 4 : 0;
  static constexpr int OFF_BAR = (OFF_MRG + MRGB + 15) / 16 * 16;
  static constexpr int NBAR = 2 * STAGES + 6;     // full, empty, ready[2], freeb[2], mrg[2]
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + ALIGN;   // + alignment slack
  static_assert(!SWZ || (OFF_V % 1024 == 0 && kStageKV % 1024 == 0 && PLANE % 1024 == 0),
                "planes on 1024-byte boundaries");
};

// Byte offset of 16-byte piece `piece` of K (or V) row `row` in a stage's
// swizzled planes: plane piece / 8, the row's 128-byte line, the piece's slot
// within the line XORed with the row's position in its group of eight (the
// layout a TMA load with a 128-byte swizzle writes at a 1024-byte aligned
// address).
__device__ __forceinline__ int swz_offset(int row, int piece, int plane_bytes) {
  return (piece >> 3) * plane_bytes + row * 128 + (((piece & 7) ^ (row & 7)) << 4);
}

// Item decode shared by the builder: item -> (b, c, g).  Items come in two
// classes: first those of the groups gorder[0 .. n_indep), then those of the
// other groups; within a class chunk by chunk, group fastest.  With a compact
// item space (B <= kMaxBatchCompact) the chunks are only those below n_b,
// chunk major over the concatenated sequences; cum[b] holds the number of
// chunks of sequences before b.  Otherwise every (b, c < nchunk) is a chunk and
// those beyond n_b are skipped.
__device__ __forceinline__ void decode_item(int item, bool compact, const int* cum, int B,
                                            int Hkv, int nchunk, int n_indep, int ncg,
                                            const uint8_t* gorder, int& b, int& c, int& g) {
  int gi, cg;
  if (item < ncg * n_indep) {
    gi = item % n_indep;
    cg = item / n_indep;
  } else {
    const int r = item - ncg * n_indep, nd = Hkv - n_indep;
    gi = n_indep + r % nd;
    cg = r / nd;
  }
  g = gorder[gi];
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

// Consumer warps for the G heads of an item, in proportion to each head's rows:
// every head with rows gets one warp, then each further warp goes to the head
// with the most rows per warp (lowest head on ties).  Warps are numbered head
// by head: asg[w] = head | slot << 4 (kNoHead when the item has no rows at all),
// nh[h] = warps of head h.  Run by one thread.
template <int G, int NW>
__device__ __forceinline__ void assign_warps(const int (&work)[G], uint8_t* asg, uint8_t* nhs) {
  int nh[G];
  int used = 0;
#pragma unroll
  for (int t = 0; t < G; ++t) {
    nh[t] = work[t] > 0 ? 1 : 0;
    used += nh[t];
  }
  if (used > 0) {
    for (; used < NW; ++used) {
      int best = -1, bw = 0, bn = 1;
#pragma unroll
      for (int t = 0; t < G; ++t) {
        if (nh[t] > 0 && (best < 0 || (long long)work[t] * bn > (long long)bw * nh[t])) {
          best = t;
          bw = work[t];
          bn = nh[t];
        }
      }
#pragma unroll
      for (int t = 0; t < G; ++t) nh[t] += (t == best) ? 1 : 0;
    }
  }
  int w = 0;
#pragma unroll
  for (int t = 0; t < G; ++t) {
    nhs[t] = (uint8_t)nh[t];
    for (int j = 0; j < nh[t]; ++j) asg[w++] = (uint8_t)(t | (j << 4));
  }
  for (; w < NW; ++w) asg[w] = kNoHead;
}

// Merge of two online-softmax states (m: running max of raw dots, l: sum of
// weights) into the first; returns the weights of the two accumulators.
struct MergeW {
  float a, b;
};
__device__ __forceinline__ MergeW merge_weights(float& m, float& l, float m2, float l2, float sl) {
  const float M = fmaxf(m, m2);
  MergeW w;
  w.a = (m == -INFINITY) ? 0.f : fast_exp2((m - M) * sl);
  w.b = (m2 == -INFINITY) ? 0.f : fast_exp2((m2 - M) * sl);
  l = l * w.a + l2 * w.b;
  m = M;
  return w;
}

template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
__device__ __forceinline__ void consumer_loop(const AttnParams& p, unsigned char* smem,
                                              uint64_t* full, uint64_t* empty, uint64_t* freeb);
template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
__device__ __forceinline__ void consumer_loop_mma(const AttnParams& p, unsigned char* smem,
                                                  uint64_t* full, uint64_t* empty, uint64_t* freeb,
                                                  uint64_t* mrg);

// The tail of a stack layer's attention kernel: the combine of the previous
// layer (its partial states are complete once the previous kernel of the stream
// has), with its sparse heads' window branch when it has one (combine_body.cuh),
// run by every CTA that has no attention item left.  Work items are whole
// (sequence, head) pairs taken from a counter.  Each of the CTA's NSL slots (a
// warp, or half a warp for d = 64) merges the states of every NSL-th chunk,
// eight states in flight, into running sums (combine_body.cuh: absorb); the
// slots are then merged in a fixed order and the head's output is written.  The
// order of the merges does not depend on scheduling.
template <typename T, int D, int NT>
__device__ __forceinline__ void tail_combine(const AttnParams& p, unsigned char* smem) {
  constexpr int LPR = D / 4;             // lanes per state row
  constexpr int SPW = 32 / LPR;          // state rows per warp
  constexpr int NSL = (NT / 32) * SPW;   // slots
  constexpr int RS = D + 4;              // slot row in shared memory: acc[D], m, l
  static_assert(NT >= D, "one thread per output element");
  float* red = reinterpret_cast<float*>(smem);
  int* s_item = reinterpret_cast<int*>(smem + NSL * RS * 4);
  float* wsm = reinterpret_cast<float*>(smem + NSL * RS * 4 + 16);   // window branch scratch
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = warp * SPW + lane / LPR, col = (lane % LPR) * 4;
  const float sl = p.scale_log2;
  for (;;) {
    if (threadIdx.x == 0) *s_item = (int)atomicAdd(p.t_counter, 1u);
    __syncthreads();
    const int bh = *s_item;
    if (bh >= p.t_heads) break;
    const int b = bh / p.Hq;
    const int n = min(max(__ldg(&p.seqlens[b]), 1), p.N_max);
    const int nc = (n + p.t_chunk - 1) / p.t_chunk;
    const int32_t* pn = p.t_part_n + (size_t)bh * p.nchunk;
    const float2* ml = reinterpret_cast<const float2*>(p.t_part_ml) + (size_t)bh * p.nchunk * kPartSlots;
    const float* pa = p.t_part_acc + (size_t)bh * p.nchunk * kPartSlots * D;
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // chunks slot, slot + NSL, ...: two at a time, four states of each in flight
    for (int ca = slot; ca < nc; ca += 2 * NSL) {
      const int cb = ca + NSL;
      const int na = min(max(__ldcg(pn + ca), 0), kPartSlots);
      const int nb = cb < nc ? min(max(__ldcg(pn + cb), 0), kPartSlots) : 0;
      for (int s0 = 0; s0 < max(na, nb); s0 += 4) {
        float2 e[8];
        float4 a[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int c = q < 4 ? ca : cb, st = s0 + (q & 3);
          e[q] = make_float2(-INFINITY, 0.f);
          a[q] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (st < (q < 4 ? na : nb)) {
            const size_t si = (size_t)c * kPartSlots + st;
            e[q] = __ldcg(ml + si);
            a[q] = __ldcg(reinterpret_cast<const float4*>(pa + si * D + col));
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) absorb(e[q], a[q], sl, m, l, acc);
      }
    }
    float* row = red + slot * RS;
    *reinterpret_cast<float4*>(row + col) = acc;
    if (col == 0) {
      row[D] = m;
      row[D + 1] = l;
    }
    __syncthreads();
    // a sparse head's window branch (every thread; fused below)
    const bool win = window_on(p.t_win, bh % p.Hq);
    float ow = 0.f;
    if (win) ow = window_out<T, D>(p.t_win, bh, p.Hq, n, sl, wsm);
    if (threadIdx.x < D) {
      float M = -INFINITY;
      for (int s2 = 0; s2 < NSL; ++s2) M = fmaxf(M, red[s2 * RS + D]);
      float A = 0.f, Lsum = 0.f;
      if (M != -INFINITY) {
        for (int s2 = 0; s2 < NSL; ++s2) {
          const float ms = red[s2 * RS + D];
          const float w = ms == -INFINITY ? 0.f : fast_exp2((ms - M) * sl);
          A = fmaf(w, red[s2 * RS + threadIdx.x], A);
          Lsum = fmaf(w, red[s2 * RS + D + 1], Lsum);
        }
      }
      float o = Lsum > 0.f ? A / Lsum : 0.f;
      if (win) o = gate_fuse(o, ow, p.t_win.gate[bh]);
      store_out<T>(reinterpret_cast<T*>(p.t_out) + (size_t)bh * D + threadIdx.x, o);
    }
    __syncthreads();   // the slot rows and the item slot are rewritten next
  }
}

template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
__global__ void __launch_bounds__((NW + NP) * 32, 1)
    attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<T, D, G, NW, NP, TT, STAGES>;
  constexpr int ROWB = C::ROWB, PPR = C::PPR, RPI = C::RPI, E = C::E, NS = C::NS;

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem =
      smem_raw + (((uint32_t)C::ALIGN - (smem_u32(smem_raw) & (C::ALIGN - 1u))) & (C::ALIGN - 1u));
  int4* info = reinterpret_cast<int4*>(smem + C::OFF_INFO);
  int* cum = reinterpret_cast<int*>(smem + C::OFF_CUM);
  // per stage: full (q and K/V rows landed; one arrival per streaming warp),
  // empty (every consumer warp is done with the stage); per item buffer: ready
  // (built), freeb (streamed and consumed: every streaming and consumer warp)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* ready = empty + STAGES;
  uint64_t* freeb = ready + 2;
  uint64_t* mrg = freeb + 2;   // consumers' item-end merge: [0] states written, [1] states read

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = p.Hq, Hkv = p.Hkv, N_max = p.N_max, B = p.B;
  const bool compact = B <= kMaxBatchCompact;
  // Programmatic dependent launch: no warp waits for the previous kernel of the
  // stream at the start.  The builder alone waits for it, before it reads the
  // first set that kernel may still be writing (the groups past n_indep) and at
  // the latest once it has claimed its last item; only then does it let the
  // next kernel launch.  So when every CTA has let the next kernel go, the
  // previous kernel has completed, and the layer before it too.
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], NS);
      mbar_init(&empty[s], NW);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ready[i], 1);
      mbar_init(&freeb[i], NS + NW);
      mbar_init(&mrg[i], NW);
    }
    fence_mbar_init();
  }
  if (warp == NW && compact) {
    // chunk counts per sequence -> exclusive prefix in cum[0..B]
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int n = b < B ? min(max(__ldg(&p.seqlens[b]), 1), N_max) : 0;
      const int nc = (n + p.chunk - 1) / p.chunk;
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

  if constexpr (C::RSPLIT) {
    if (warp >= NW) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::PREGS));
    else asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::CREGS));
  }
  if (warp == NW + 1) {
    // ------------------------------------------------------------ builder
    const int ncg = compact ? cum[B] : B * p.nchunk_run;   // (sequence, chunk) pairs
    const int n_items = ncg * Hkv;
    const int first_dep = ncg * p.n_indep;                   // first item of a waiting group
    bool waited = false, released = false;                   // warp-uniform
    auto wait_prev = [&]() {
      if (!waited) {
        pdl_wait();
        waited = true;
      }
    };
    // claim an item (lane 0) and load what building its row list needs
    auto claim = [&]() -> int { return lane == 0 ? (int)atomicAdd(p.counter, 1u) : 0; };
    auto prefetch = [&](int item, int& nraw, uint32_t (&w)[G]) {
      nraw = 1;
#pragma unroll
      for (int t = 0; t < G; ++t) w[t] = 0u;
      if (item >= n_items) {
        // this CTA takes no further item
        wait_prev();
        if (!released) {
          pdl_launch_dependents();
          released = true;
        }
        return;
      }
      if (item >= first_dep) wait_prev();
      int b, c, g;
      decode_item(item, compact, cum, B, Hkv, p.nchunk_run, p.n_indep, ncg, p.gorder, b, c, g);
      nraw = __ldg(&p.seqlens[b]);
      const int word = c * (p.chunk / 32) + lane;
      if (lane < p.chunk / 32 && word < p.nwords) {
        // sparse heads' words only (a retrieval head reads every row), through
        // L2: in a stack the previous kernel may have rewritten these rows
        // while this kernel ran
        const size_t wbase = (size_t)(b * Hq + g * G) * p.nwords + word;
#pragma unroll
        for (int t = 0; t < G; ++t) {
          const int h = g * G + t;
          if (!((p.role[h >> 5] >> (h & 31)) & 1u)) w[t] = __ldcg(&p.bitmaps[wbase + (size_t)t * p.nwords]);
        }
      }
    };
    if (blockIdx.x == 0) {
      for (int bb = lane; bb < B; bb += 32) {
        const int n_raw = __ldg(&p.seqlens[bb]);
        if (n_raw < 1 || n_raw > N_max) flag_error(p.err, kErrBadSeqlen);
        if (p.k_per_seq && __ldg(&p.k_per_seq[bb]) < 1) flag_error(p.err, kErrBadBudget);
      }
    }
    int cur = __shfl_sync(kFull, claim(), 0), cur_n = 1;
    uint32_t cur_w[G];
    prefetch(cur, cur_n, cur_w);
    int claimed = claim();
    for (uint32_t it = 0;; ++it) {
      const int buf = it & 1;
      if (!mbar_wait(&freeb[buf], ((it >> 1) & 1u) ^ 1u, p.err, p.wait_ns)) break;
      unsigned char* ib = smem + C::OFF_ITEM + buf * C::IBUF;
      int* desc = reinterpret_cast<int*>(ib);
      uint8_t* asg = ib + C::IB_ASG;
      int32_t* lpos = reinterpret_cast<int32_t*>(ib + C::IB_LPOS);
      int total = 0, b = 0, c = 0, g = 0, p0 = 0;
      uint32_t rmask = 0;
      for (;;) {   // skip chunks beyond n_b (only without the compact space)
        if (cur >= n_items) {
          total = -1;
          break;
        }
        decode_item(cur, compact, cum, B, Hkv, p.nchunk_run, p.n_indep, ncg, p.gorder, b, c, g);
        const int n = min(max(cur_n, 1), N_max);
        p0 = c * p.chunk;
        const int h0 = g * G;
        // claim and load the item after this one while this one is built
        int nxt_n = 1;
        uint32_t nxt_w[G];
        const int nxt = __shfl_sync(kFull, claimed, 0);
        prefetch(nxt, nxt_n, nxt_w);
        claimed = claim();
        if (p0 < n) {
          const int p1 = min(p0 + p.chunk, n);
          rmask = 0;
#pragma unroll
          for (int t = 0; t < G; ++t) rmask |= ((p.role[(h0 + t) >> 5] >> ((h0 + t) & 31)) & 1u) << t;
          const int nwords = (p1 - p0 + 31) >> 5;
          const int nbits = lane < nwords ? min(32, p1 - p0 - 32 * lane) : 0;
          const uint32_t valid = nbits >= 32 ? kFull : ((1u << nbits) - 1u);
          uint32_t bits[G];
          uint32_t uni = 0;
#pragma unroll
          for (int t = 0; t < G; ++t) {
            bits[t] = ((rmask >> t) & 1u) ? valid : (cur_w[t] & valid);
            uni |= bits[t];
          }
          const int cnt = __popc(uni);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
          }
          total = __shfl_sync(kFull, incl, 31);
          const int ubase = incl - cnt;      // union index of this word's first row
          if (rmask == 0) {
            // sparse item: positions of the union rows, in order
            int o = ubase;
            uint32_t u = uni;
            while (u) {
              const int j = __ffs(u) - 1;
              u &= u - 1;
              lpos[o++] = p0 + 32 * lane + j;
            }
          }
          if constexpr (C::MMA) {
            // the heads' membership words (a retrieval head's: every valid row)
            if (lane < p.chunk / 32) {
              uint32_t hv[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) hv[t] = t < G ? bits[t] : 0u;
              uint4* hw = reinterpret_cast<uint4*>(ib + C::IB_HW) + 2 * lane;
              hw[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
              hw[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
            // the consumer warps' states are merged into one per head
            if (lane < G) p.part_n[(size_t)(b * Hq + h0 + lane) * p.nchunk + c] = 1;
          } else {
            // each sparse head's rows as union indices, in order (lane w places
            // the rows of word w), and where each tile starts in that list: a
            // tile boundary (a multiple of TT > 32 union rows) falls inside at
            // most one word, whose lane writes the start (a retrieval head takes
            // every row: no list)
            uint16_t* hrow = reinterpret_cast<uint16_t*>(ib + C::IB_HROW);
            uint16_t* tst = reinterpret_cast<uint16_t*>(ib + C::IB_TST);
            const int ntile = (total + TT - 1) / TT;
            const int tb = (ubase + TT - 1) / TT;         // first tile starting at or after ubase
            const bool has_bound = tb * TT < ubase + cnt;  // ... and inside this word
            int bpos = 0;                                  // position of that boundary row
            if (has_bound) {
              uint32_t u = uni;
              for (int r2 = tb * TT - ubase; r2 > 0; --r2) u &= u - 1;
              bpos = __ffs(u) - 1;
            }
            int work[G];
#pragma unroll
            for (int t = 0; t < G; ++t) {
              const int ct = __popc(bits[t]);
              int ic = ct;
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, ic, o);
                if (lane >= o) ic += y;
              }
              work[t] = __shfl_sync(kFull, ic, 31);
              if ((rmask >> t) & 1u) continue;
              uint16_t* hl = hrow + t * kChunk;
              int k = ic - ct;
              uint32_t u = bits[t];
              while (u) {
                const int j = __ffs(u) - 1;
                u &= u - 1;
                hl[k++] = (uint16_t)(ubase + __popc(uni & ((1u << j) - 1u)));
              }
              uint16_t* ts = tst + t * 32;
              if (has_bound) ts[tb] = (uint16_t)(ic - ct + __popc(bits[t] & ((1u << bpos) - 1u)));
              if (lane == 0) {
                ts[0] = 0;
                ts[ntile] = (uint16_t)work[t];
              }
            }
            if (lane == 0) assign_warps<G, NW>(work, asg, asg + NW);
            __syncwarp();
            // partial states each head's warps will write for this chunk
            if (lane < G)
              p.part_n[(size_t)(b * Hq + h0 + lane) * p.nchunk + c] = (int)asg[NW + lane];
          }
        }
        cur = nxt;
        cur_n = nxt_n;
#pragma unroll
        for (int t = 0; t < G; ++t) cur_w[t] = nxt_w[t];
        if (p0 < n) break;
      }
      if (lane == 0) {
        desc[0] = total;
        desc[1] = b;
        desc[2] = c;
        desc[3] = g;
        desc[4] = p0;
        desc[5] = (int)rmask;
      }
      __syncwarp();
      // (test only: with p.withhold_first the first item is never announced,
      // so every wait that depends on it runs out after p.wait_ns)
      if (lane == 0 && !(p.withhold_first && it == 0)) mbar_arrive(&ready[buf]);
      if (total < 0) break;
    }
    wait_prev();   // (a wait that gave up leaves the loop early)
    if (!released) pdl_launch_dependents();
  } else if (warp >= NW) {
    // ------------------------------------------------------ streaming warps
    const int sw = warp == NW ? 0 : warp - NW - 1;   // 0: publishes tiles, bulk copies
    const uint64_t pol = l2_evict_first_policy();
    const bool tma_rows = C::TMA_ROWS > 0 && NS > 1 && p.gather_tma != 0;
    uint32_t s = 0, ph = 0;                // ring stage and its phase parity
    bool ok = true;
    for (uint32_t it = 0;; ++it) {
      const int buf = it & 1;
      if (!mbar_wait(&ready[buf], (it >> 1) & 1u, p.err, p.wait_ns)) break;
      const unsigned char* ib = smem + C::OFF_ITEM + buf * C::IBUF;
      const int* desc = reinterpret_cast<const int*>(ib);
      const int32_t* lpos = reinterpret_cast<const int32_t*>(ib + C::IB_LPOS);
      const int total = desc[0], b = desc[1], c = desc[2], g = desc[3], p0 = desc[4];
      const uint32_t rmask = (uint32_t)desc[5];
      const bool dense = rmask != 0;
      const int h0 = g * G;
      const int unit = b * Hkv + g;
      const T* kbase = reinterpret_cast<const T*>(p.k) + (size_t)unit * N_max * D;
      const T* vbase = reinterpret_cast<const T*>(p.v) + (size_t)unit * N_max * D;
      const int row0 = unit * N_max;        // this group's first row in the tensor maps
      // the end is one entry; a chunk no head of the group uses is one empty tile
      const int ntile = total <= 0 ? 1 : (total + TT - 1) / TT;
      for (int tt = 0; tt < ntile; ++tt) {
        const int t0 = tt * TT;
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        const int nrows = total < 0 ? 0 : min(TT, total - t0);
        const int flags = total < 0 ? kTerm
                                    : ((t0 == 0 ? kFirst : 0) | (t0 + TT >= total ? kLast : 0) |
                                       (dense ? kDense : 0));
        unsigned char* kd = smem + C::OFF_K + s * C::kStageKV;
        unsigned char* vd = smem + C::OFF_V + s * C::kStageKV;
        const bool gather = !(flags & (kDense | kTerm));
        if (sw == 0 && lane == 0) {
          info[2 * s] = make_int4(b, h0, c, nrows);
          info[2 * s + 1] = make_int4(flags, (int)rmask, t0, buf | (tt << 8));
        }
        // rows [0, nt) by TMA (whole groups of four, the last one padded only
        // when it ends the tile), rows [nt, nrows) by 16-byte copies
        const int nt = !gather || !tma_rows
                           ? 0
                           : (nrows <= 4 ? nrows : ((nrows * C::TMA_ROWS) >> 4) & ~3);
        const int ngrp = (nt + 3) >> 2;
        const int csw = tma_rows ? sw - 1 : sw, ncs = tma_rows ? NS - 1 : NS;
        if (gather && csw >= 0) {
          // 16-byte copies shared by the copying warps, each lane's copies
          // tracked by the stage's full barrier
          for (int r0 = nt + csw * RPI; r0 < nrows; r0 += ncs * RPI) {
#pragma unroll
            for (int pc2 = 0; pc2 < (PPR + 31) / 32; ++pc2) {
              const int row = r0 + (PPR >= 32 ? 0 : lane / PPR);
              const int piece = PPR >= 32 ? pc2 * 32 + lane : lane % PPR;
              if (row < nrows && piece < PPR) {
                const size_t src = (size_t)lpos[t0 + row] * D + piece * E;
                const int dst = C::SWZ ? swz_offset(row, piece, C::PLANE) : row * ROWB + piece * 16;
                cp_async16(kd + dst, kbase + src);
                cp_async16(vd + dst, vbase + src);
              }
            }
          }
          cp_async_mbar_arrive(&full[s]);
        }
        __syncwarp();
        if (lane == 0 && sw != 0) mbar_arrive(&full[s]);
        if (lane == 0 && sw == 0) {
          // swizzled planes: a dense tile comes as whole boxes (TT rows, or
          // 16-row boxes covering a shorter tile)
          const uint32_t drows = !C::SWZ ? (uint32_t)nrows
                                         : (nrows == TT ? (uint32_t)TT : (uint32_t)((nrows + 15) & ~15));
          const uint32_t bytes = ((flags & kDense) ? 2u * drows * ROWB : 0u) +
                                 ((flags & kFirst) ? (uint32_t)C::kQBytes : 0u) +
                                 2u * (uint32_t)ngrp * 4u * ROWB;
          fence_proxy_async_smem();
          if (bytes) mbar_arrive_expect_tx(&full[s], bytes);
          else mbar_arrive(&full[s]);
          if (flags & kFirst) {
            T* qd = reinterpret_cast<T*>(smem + C::OFF_Q + s * C::QSTRIDE);
            bulk_g2s(qd, reinterpret_cast<const T*>(p.q) + (size_t)(b * Hq + h0) * D,
                     (uint32_t)C::kQBytes, &full[s], pol);
          }
          if (flags & kDense) {
            if constexpr (C::SWZ) {
              // per plane, K then V: one TT-row box, or 16-row boxes
#pragma unroll
              for (int pl = 0; pl < C::NPL; ++pl) {
                const int po = pl * C::PLANE;
                if (nrows == TT) {
                  tma_load_3d(kd + po, &p.tmk_tile, 64 * pl, p0 + t0, unit, &full[s], pol);
                  tma_load_3d(vd + po, &p.tmv_tile, 64 * pl, p0 + t0, unit, &full[s], pol);
                } else {
                  for (int i = 0; i < nrows; i += 16) {
                    tma_load_3d(kd + po + i * 128, &p.tmk_rest, 64 * pl, p0 + t0 + i, unit, &full[s], pol);
                    tma_load_3d(vd + po + i * 128, &p.tmv_rest, 64 * pl, p0 + t0 + i, unit, &full[s], pol);
                  }
                }
              }
            } else {
              const size_t off = (size_t)(p0 + t0) * D;
              bulk_g2s(kd, kbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
              bulk_g2s(vd, vbase + off, (uint32_t)nrows * ROWB, &full[s], pol);
            }
          }
        }
        if (!C::SWZ && ngrp > 0 && sw == 0) {
          // four rows per copy; a padded group repeats the range's last row
          const int last = lpos[t0 + nt - 1];
          for (int gi = lane; gi < ngrp; gi += 32) {
            const int4 q4 = *reinterpret_cast<const int4*>(lpos + t0 + 4 * gi);
            const int y0 = row0 + q4.x;
            const int y1 = row0 + (4 * gi + 1 < nt ? q4.y : last);
            const int y2 = row0 + (4 * gi + 2 < nt ? q4.z : last);
            const int y3 = row0 + (4 * gi + 3 < nt ? q4.w : last);
            tma_gather4(kd + gi * 4 * ROWB, &p.tmk, 0, y0, y1, y2, y3, &full[s], pol);
            tma_gather4(vd + gi * 4 * ROWB, &p.tmv, 0, y0, y1, y2, y3, &full[s], pol);
          }
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok || total < 0) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&freeb[buf]);   // done reading this item's positions
    }
  } else if (warp < NW) {
    if constexpr (C::MMA) consumer_loop_mma<T, D, G, NW, NP, TT, STAGES>(p, smem, full, empty, freeb, mrg);
    else consumer_loop<T, D, G, NW, NP, TT, STAGES>(p, smem, full, empty, freeb);
  }
  __syncthreads();
  if (p.t_heads > 0) {
    if constexpr (C::RSPLIT) {
      // back to the launch's registers per thread in every warp
      if (warp >= NW) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::LREGS));
      else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::LREGS));
    }
    pdl_wait();   // the previous layer's partial states are complete
    static_assert((C::NT / 32) * (32 / (D / 4)) * (D + 4) * 4 + 16 + window_smem_floats<D>() * 4 <=
                      C::OFF_INFO,
                  "the tail's shared memory fits the (drained) ring");
    tail_combine<T, D, C::NT>(p, smem);
  }
  // ---- the last CTA to leave resets the launch counters for the next launch
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.exits, 1u) == gridDim.x - 1) {
      *p.counter = 0u;
      *p.t_counter = 0u;
      *p.exits = 0u;
      __threadfence();
    }
  }
}

// Consumer warps of attn_kernel (see the file comment).
template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
__device__ __forceinline__ void consumer_loop(const AttnParams& p, unsigned char* smem,
                                              uint64_t* full, uint64_t* empty, uint64_t* freeb) {
  using C = AttnCfg<T, D, G, NW, NP, TT, STAGES>;
  constexpr int E = C::E, DL = C::DL, CPL = C::CPL, ROWB = C::ROWB;
  constexpr int ILP = ilp_of<T, D>();
  const int4* info = reinterpret_cast<const int4*>(smem + C::OFF_INFO);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane / kLanesPerPair, pp = lane % kLanesPerPair;   // pair slot, quarter
  // Chunk order rotated per lane: a 16-byte shared load is served per group of
  // 8 consecutive lanes (slots r, r+1 with r even, all four quarters), which
  // must touch 8 different 16-byte bank slots of a 128-byte line.  The rotation
  // depends on r only through r & 1 (slots r, r^2, r^4 share it), and slot r^1
  // is rotated by exactly CPL/2 chunks against slot r.
  const int rot = CPL == 2 ? (r & 1)
                : CPL == 4 ? ((pp >> 1) + 2 * (r & 1)) % 4
                           : (pp + 4 * (r & 1)) % CPL;
  const float sl = p.scale_log2;
  const float lazy = kLazyLog2 / sl;      // raw-dot growth that moves the maximum

  int coff[CPL];                           // byte offsets of the lane's chunks in a row
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) coff[cc] = pp * DL * (int)sizeof(T) + ((cc + rot) % CPL) * 16;

  float2 qr[CPL][E / 2];
  float2 acc[CPL][E / 2];
  float m = -INFINITY, mth = -INFINITY, msl = 0.f, l = 0.f;
  int myh = -1, slot = 0, nh = 1, buf = 0;
  int kfirst = 0;                          // first batch of this tile for the warp

  bool ident = false, lg_on = false;
  float* lg = nullptr;
  int b = 0, h0 = 0, c = 0;

  uint32_t s = 0, ph = 0;
  for (;;) {
    if (!mbar_wait(&full[s], ph, p.err, p.wait_ns)) break;
    const int4 i0 = info[2 * s], i1 = info[2 * s + 1];
    const int flags = i1.x;
    if (flags & kTerm) break;
    const int nrows = i0.w, t0 = i1.z, tt = i1.w >> 8;
    const unsigned char* ib = smem + C::OFF_ITEM + (i1.w & 1) * C::IBUF;

    if (flags & kFirst) {
      b = i0.x;
      h0 = i0.y;
      c = i0.z;
      buf = i1.w & 1;
      const uint8_t a = ib[C::IB_ASG + warp];
      myh = a == kNoHead ? -1 : (a & 15);
      slot = a >> 4;
      kfirst = slot;
      if (myh >= 0) {
        nh = ib[C::IB_ASG + NW + myh];
        ident = (i1.y >> myh) & 1;
        lg_on = ident && pp == 0;
        lg = p.logits + (size_t)(b * p.Hq + h0 + myh) * p.N_max + (size_t)c * p.chunk;
        const unsigned char* qs = smem + C::OFF_Q + s * C::QSTRIDE + myh * ROWB;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          Vec<T>::load16(qs + coff[cc], qr[cc]);
#pragma unroll
          for (int e = 0; e < E / 2; ++e) acc[cc][e] = make_float2(0.f, 0.f);
        }
      }
      m = -INFINITY;
      mth = -INFINITY;
      msl = 0.f;
      l = 0.f;
    }

    if (myh >= 0) {
      // this tile's rows of the warp's head: all of them for a retrieval head,
      // else a slice of the head's row list (union indices of the item)
      int cnt = nrows, st0 = 0;
      const uint16_t* hl = reinterpret_cast<const uint16_t*>(ib + C::IB_HROW) + myh * kChunk;
      if (!ident) {
        const uint16_t* ts = reinterpret_cast<const uint16_t*>(ib + C::IB_TST) + myh * 32;
        st0 = ts[tt];
        cnt = (int)ts[tt + 1] - st0;
      }
      const int nb = (cnt + kPairsPerBatch - 1) / kPairsPerBatch;
      const unsigned char* kt = smem + C::OFF_K + s * C::kStageKV;
      const unsigned char* vt = smem + C::OFF_V + s * C::kStageKV;
      // batch k is served by slot (k + tt) % nh: the first batch of a tile
      // moves from slot to slot so that no warp of the head always gets the most
      int k = kfirst;
      kfirst = kfirst == 0 ? nh - 1 : kfirst - 1;
      // NBAT batches per iteration (k, k + nh, ...) so that their dependency
      // chains overlap; batches past the last are empty (no pair taken).  A
      // retrieval head fills whole tiles, so its warps take ILP batches at
      // once; a sparse head's warps get about two batches per tile, so one.
      auto run = [&](auto nbat_tag) {
      constexpr int NBAT = decltype(nbat_tag)::value;
      for (; k < nb; k += NBAT * nh) {
        int rowu[NBAT];
        bool validu[NBAT];
        uint4 raw[NBAT][CPL];
        float svu[NBAT];
        // ---- rows and K chunks
#pragma unroll
        for (int u = 0; u < NBAT; ++u) {
          const int idx = (k + u * nh) * kPairsPerBatch + r;
          validu[u] = idx < cnt;
          rowu[u] = validu[u] ? (ident ? idx : (int)hl[st0 + idx] - t0) : 0;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
            raw[u][cc] = *reinterpret_cast<const uint4*>(kt + rowu[u] * ROWB + coff[cc]);
        }
        // ---- q.K over the lane's quarter: CPL independent partial sums
#pragma unroll
        for (int u = 0; u < NBAT; ++u) {
          float2 part[CPL];
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) {
            float2 kx[E / 2];
            Vec<T>::widen(raw[u][cc], kx);
            part[cc] = __fmul2_rn(qr[cc][0], kx[0]);
#pragma unroll
            for (int e = 1; e < E / 2; ++e) part[cc] = __ffma2_rn(qr[cc][e], kx[e], part[cc]);
          }
#pragma unroll
          for (int w2 = 1; w2 < CPL; w2 <<= 1)
#pragma unroll
            for (int cc = 0; cc + w2 < CPL; cc += 2 * w2)
              part[cc] = __fadd2_rn(part[cc], part[cc + w2]);
          svu[u] = part[0].x + part[0].y;
        }
        // ---- V chunks of the same rows (row 0 always holds real data; a pair
        // that is not taken gets weight 0), loaded while the scores finish
#pragma unroll
        for (int u = 0; u < NBAT; ++u)
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
            raw[u][cc] = *reinterpret_cast<const uint4*>(vt + rowu[u] * ROWB + coff[cc]);
        float mx = -INFINITY;
#pragma unroll
        for (int u = 0; u < NBAT; ++u) {
          float dot = svu[u];
          dot += __shfl_xor_sync(kFull, dot, 1);
          dot += __shfl_xor_sync(kFull, dot, 2);
          if (lg_on && validu[u]) lg[t0 + rowu[u]] = dot;
          svu[u] = validu[u] ? dot : -INFINITY;
          mx = fmaxf(mx, svu[u]);
        }
        // ---- online softmax with a lazy maximum (warp-uniform branch)
        if (__any_sync(kFull, mx > mth)) {
          const float mn = mx > mth ? mx : m;
          const float al = (mn == m) ? 1.f : fast_exp2((m - mn) * sl);   // 0 while m is -inf
          const float2 a2 = make_float2(al, al);
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
            for (int e = 0; e < E / 2; ++e) acc[cc][e] = __fmul2_rn(acc[cc][e], a2);
          l *= al;
          m = mn;
          mth = (m == -INFINITY) ? -INFINITY : m + lazy;
          msl = (m == -INFINITY) ? 0.f : m * sl;
        }
        // ---- P.V on the same rows and quarter
#pragma unroll
        for (int u = 0; u < NBAT; ++u) {
          const float pr = fast_exp2(fmaf(svu[u], sl, -msl));   // 0 for rows not taken
          l += pr;
          const float2 p2 = make_float2(pr, pr);
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) {
            float2 vx[E / 2];
            Vec<T>::widen(raw[u][cc], vx);
#pragma unroll
            for (int e = 0; e < E / 2; ++e) acc[cc][e] = __ffma2_rn(p2, vx[e], acc[cc][e]);
          }
        }
      }
      };
      if (ident) run(std::integral_constant<int, ILP>{});
      else run(std::integral_constant<int, 1>{});
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == STAGES) {
      s = 0;
      ph ^= 1u;
    }

    if (flags & kLast) {
      if (lane == 0) mbar_arrive(&freeb[buf]);   // done with this item's buffer
      if (myh >= 0) {
        // ---- merge the warp's eight slots in registers: r^2, r^4 (same
        // rotation), then r^1 (rotated by CPL/2 chunks)
#pragma unroll
        for (int o = 2 * kLanesPerPair; o <= 4 * kLanesPerPair; o <<= 1) {
          const MergeW w = merge_weights(m, l, __shfl_xor_sync(kFull, m, o),
                                         __shfl_xor_sync(kFull, l, o), sl);
          const float2 wa = make_float2(w.a, w.a), wb = make_float2(w.b, w.b);
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
              float2 x;
              x.x = __shfl_xor_sync(kFull, acc[cc][e].x, o);
              x.y = __shfl_xor_sync(kFull, acc[cc][e].y, o);
              acc[cc][e] = __ffma2_rn(acc[cc][e], wa, __fmul2_rn(x, wb));
            }
        }
        {
          constexpr int o = kLanesPerPair;
          const MergeW w = merge_weights(m, l, __shfl_xor_sync(kFull, m, o),
                                         __shfl_xor_sync(kFull, l, o), sl);
          const float2 wa = make_float2(w.a, w.a), wb = make_float2(w.b, w.b);
          float2 x[CPL][E / 2];
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
              x[cc][e].x = __shfl_xor_sync(kFull, acc[(cc + CPL / 2) % CPL][e].x, o);
              x[cc][e].y = __shfl_xor_sync(kFull, acc[(cc + CPL / 2) % CPL][e].y, o);
            }
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
            for (int e = 0; e < E / 2; ++e)
              acc[cc][e] = __ffma2_rn(acc[cc][e], wa, __fmul2_rn(x[cc][e], wb));
        }
        // ---- slot 0 (lanes 0..3) writes the warp's state to its partial slot
        if (r == 0) {
          const size_t ps = ((size_t)(b * p.Hq + h0 + myh) * p.nchunk + c) * kPartSlots + slot;
          float* dst = p.part_acc + ps * D + pp * DL;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
            for (int e = 0; e < E / 2; e += 2)
              *reinterpret_cast<float4*>(dst + ((cc + rot) % CPL) * E + 2 * e) =
                  make_float4(acc[cc][e].x, acc[cc][e].y, acc[cc][e + 1].x, acc[cc][e + 1].y);
          if (pp == 0) *reinterpret_cast<float2*>(p.part_ml + ps * 2) = make_float2(m, l);
        }
      }
    }
  }
}

// ---- tensor-core consumers (bf16 caches) -------------------------------------
// D += A * B on one warp: A 16x16 bf16 (row-major fragments), B 16x8 bf16
// (column fragments), D and C 16x8 fp32.  Lane (g = lane / 4, t = lane % 4)
// holds A rows g, g + 8 at columns 2t, 2t + 1 and 2t + 8, 2t + 9; B rows 2t,
// 2t + 1 and 2t + 8, 2t + 9 of column g; C rows g, g + 8 at columns 2t, 2t + 1.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Transpose of an 8x8 matrix of 16-bit elements held one row per four lanes
// (lane g * 4 + t: row g, columns 2t, 2t + 1).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Consumer warps of attn_kernel for bf16 caches.  A warp takes whole slabs of
// 16 rows of a tile (slab sigma of an item, counted over its tiles, goes to warp
// sigma mod NW) and serves every head of the group on them at once:
//   S^T (16 rows x 8 heads; heads >= G are zero columns) = K_slab . q^T on the
//   tensor cores, bf16 operands and fp32 accumulation, K's fragments by
//   ldmatrix from the swizzled K planes, q's from the stage's q rows;
//   rows a head does not use (the heads' membership words of the item), rows
//   past the tile and padding heads get score -inf; retrieval heads' raw scores go to the logits;
//   online softmax per head with the lazy maximum;
//   O^T (d x 8 heads) += V_slab^T . P on the tensor cores, P rounded to bf16
//   (the weights summed into l are the rounded ones): V^T's fragments come
//   from the swizzled V planes by transposing ldmatrix, P's by two 8x8
//   transposes in registers.  Every ldmatrix is conflict-free: the eight rows
//   of a matrix sit in eight different 16-byte slots.
// At the end of an item the warps' states of each head are merged in shared
// memory (a fixed order: warp 0 first) and one state per head goes to slot 0
// of the workspace, a quarter of the partial-state traffic of one per warp.
template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
__device__ __forceinline__ void consumer_loop_mma(const AttnParams& p, unsigned char* smem,
                                                  uint64_t* full, uint64_t* empty, uint64_t* freeb,
                                                  uint64_t* mrg) {
  using C = AttnCfg<T, D, G, NW, NP, TT, STAGES>;
  constexpr int ROWB = C::ROWB;
  constexpr int NPB = D / 32;            // 32-dimension blocks
  constexpr int SPT = TT / 16;           // slabs per tile
  constexpr uint32_t kAll = (1u << G) - 1u;
  const int4* info = reinterpret_cast<const int4*>(smem + C::OFF_INFO);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int hx = 2 * t, hy = 2 * t + 1;  // the lane's two heads (columns of S^T, O^T)
  const float sl = p.scale_log2;
  const float lazy = kLazyLog2 / sl;

  uint32_t qb[2 * NPB][2];               // B fragments of q^T: head g, dims 16kk + 2t (+ 8), + 1
  float o[2 * NPB][4];                   // O^T fragments, block 2P + jp
  float m[2], mth[2], msl[2], l[2];      // per lane head (hx, hy)
  uint32_t rm = 0;
  int b = 0, h0 = 0, c = 0, buf = 0;

  uint32_t s = 0, ph = 0, mph = 0;   // ring stage and phase; merge barriers' phase
  for (;;) {
    if (!mbar_wait(&full[s], ph, p.err, p.wait_ns)) break;
    const int4 i0 = info[2 * s], i1 = info[2 * s + 1];
    const int flags = i1.x;
    if (flags & kTerm) break;
    const int nrows = i0.w, t0 = i1.z, tt = i1.w >> 8;
    const unsigned char* ib = smem + C::OFF_ITEM + (i1.w & 1) * C::IBUF;

    if (flags & kFirst) {
      b = i0.x;
      h0 = i0.y;
      c = i0.z;
      buf = i1.w & 1;
      rm = (uint32_t)i1.y;
      const uint32_t* qs =
          reinterpret_cast<const uint32_t*>(smem + C::OFF_Q + s * C::QSTRIDE + g * ROWB) + t;
#pragma unroll
      for (int kk = 0; kk < 2 * NPB; ++kk) {
        qb[kk][0] = g < G ? qs[8 * kk] : 0u;
        qb[kk][1] = g < G ? qs[8 * kk + 4] : 0u;
      }
#pragma unroll
      for (int k = 0; k < 2 * NPB; ++k) o[k][0] = o[k][1] = o[k][2] = o[k][3] = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        m[e] = -INFINITY;
        mth[e] = -INFINITY;
        msl[e] = 0.f;
        l[e] = 0.f;
      }
    }

    const bool masked = rm != kAll;       // some head of the group uses only some rows
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(ib + C::IB_HW) + 2 * t;
    const int32_t* lpos = reinterpret_cast<const int32_t*>(ib + C::IB_LPOS) + t0;
    // bit 0 / 1: head hx / hy uses union row r of this tile (a group with a
    // retrieval head reads every position of the chunk in order)
    auto lane_heads = [&](int r) -> uint32_t {
      const int po = rm ? t0 + r : lpos[r] - c * p.chunk;
      const uint2 w = *reinterpret_cast<const uint2*>(hw + (po >> 5) * 8);
      return ((w.x >> (po & 31)) & 1u) | (((w.y >> (po & 31)) & 1u) << 1);
    };
    const uint32_t lane_all = (hx < G ? 1u : 0u) | (hy < G ? 2u : 0u);
    const uint32_t kt_u32 = smem_u32(smem + C::OFF_K + s * C::kStageKV);
    const uint32_t vt_u32 = smem_u32(smem + C::OFF_V + s * C::kStageKV);
    const int nsl = (nrows + 15) >> 4;
    int j = (warp - (tt * SPT) % NW) % NW;
    if (j < 0) j += NW;
    for (; j < nsl; j += NW) {
      const int rA = 16 * j + g, rB = rA + 8;
      const bool vA = rA < nrows, vB = rB < nrows;
      // which of the lane's heads use its two rows (looked up while K loads)
      const uint32_t mkA = vA ? (masked ? lane_heads(rA) : lane_all) : 0u;
      const uint32_t mkB = vB ? (masked ? lane_heads(rB) : lane_all) : 0u;
      // A fragments of the K slab, block kk (dimensions 16kk .. + 15) from four
      // 8x8 matrices, lanes 8i .. 8i + 7 addressing matrix i: rows 8 (i % 2)
      // .. + 7 of the slab, dimensions 16kk + 8 (i / 2) .. + 7 (a row past the
      // tile reads row 0 instead; its score is masked)
      uint32_t KF[2 * NPB][4];
      {
        const int lr = 16 * j + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int rr = lr < nrows ? lr : 0;
        const uint32_t ra = kt_u32 + rr * 128;
        const int hi = lane >> 4;
#pragma unroll
        for (int kk = 0; kk < 2 * NPB; ++kk)
          ldsm_x4(ra + (kk >> 2) * C::PLANE + (((((2 * kk) & 7) + hi) ^ (rr & 7)) << 4),
                  KF[kk][0], KF[kk][1], KF[kk][2], KF[kk][3]);
      }
      // ---- S^T = K q^T (four accumulation chains)
      float sc[4][4] = {};
#pragma unroll
      for (int kk = 0; kk < 2 * NPB; ++kk)
        mma_16816(sc[kk & 3], KF[kk][0], KF[kk][1], KF[kk][2], KF[kk][3], qb[kk][0], qb[kk][1]);
      // V of the same rows, loaded while the scores finish
      // straight into A fragments of V^T: block m (dimensions 16m .. 16m + 15)
      // from four 8x8 matrices, lanes 8i .. 8i + 7 addressing matrix i: rows
      // 8 (i / 2) .. + 7 of the slab, dimensions 16m + 8 (i % 2) .. + 7 (a row
      // past the tile reads row 0 instead; its weight is 0)
      uint32_t VF[2 * NPB][4];
      {
        const int lr = 16 * j + ((lane >> 4) << 3) + (lane & 7);
        const int rr = lr < nrows ? lr : 0;
        const uint32_t ra = vt_u32 + rr * 128;
        const int hi = (lane >> 3) & 1;
#pragma unroll
        for (int mb = 0; mb < 2 * NPB; ++mb)
          ldsm_x4_trans(ra + (mb >> 2) * C::PLANE + (((((2 * mb) & 7) + hi) ^ (rr & 7)) << 4),
                        VF[mb][0], VF[mb][1], VF[mb][2], VF[mb][3]);
      }
      // raw scores: (rA, hx), (rA, hy), (rB, hx), (rB, hy)
      float sv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) sv[e] = (sc[0][e] + sc[2][e]) + (sc[1][e] + sc[3][e]);
      if (rm) {
        // retrieval heads' raw scores for the top-k (union index = position here)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * t + e;
          if (h < G && ((rm >> h) & 1u)) {
            float* lg = p.logits + (size_t)(b * p.Hq + h0 + h) * p.N_max + (size_t)c * p.chunk + t0;
            if (vA) lg[rA] = sv[e];
            if (vB) lg[rB] = sv[2 + e];
          }
        }
      }
      sv[0] = (mkA & 1u) ? sv[0] : -INFINITY;
      sv[1] = (mkA & 2u) ? sv[1] : -INFINITY;
      sv[2] = (mkB & 1u) ? sv[2] : -INFINITY;
      sv[3] = (mkB & 2u) ? sv[3] : -INFINITY;
      // ---- online softmax per head, lazy maximum (warp-uniform branch): a
      // head's maximum over the slab exceeds its threshold iff one of its
      // scores does, so the maximum itself is reduced only when it is used
      float mx[2] = {fmaxf(sv[0], sv[2]), fmaxf(sv[1], sv[3])};
      if (__any_sync(kFull, mx[0] > mth[0] || mx[1] > mth[1])) {
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          mx[0] = fmaxf(mx[0], __shfl_xor_sync(kFull, mx[0], o2));
          mx[1] = fmaxf(mx[1], __shfl_xor_sync(kFull, mx[1], o2));
        }
        float al[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float mn = mx[e] > mth[e] ? mx[e] : m[e];
          al[e] = (mn == m[e]) ? 1.f : fast_exp2((m[e] - mn) * sl);   // 0 while m is -inf
          l[e] *= al[e];
          m[e] = mn;
          mth[e] = (mn == -INFINITY) ? -INFINITY : mn + lazy;
          msl[e] = (mn == -INFINITY) ? 0.f : mn * sl;
        }
#pragma unroll
        for (int k = 0; k < 2 * NPB; ++k) {
          o[k][0] *= al[0];
          o[k][2] *= al[0];
          o[k][1] *= al[1];
          o[k][3] *= al[1];
        }
      }
      const uint32_t pa = pack_bf16(fast_exp2(fmaf(sv[0], sl, -msl[0])),
                                    fast_exp2(fmaf(sv[1], sl, -msl[1])));
      const uint32_t pb = pack_bf16(fast_exp2(fmaf(sv[2], sl, -msl[0])),
                                    fast_exp2(fmaf(sv[3], sl, -msl[1])));
      {
        const float2 fa = bf16x2_to_float2(pa), fb = bf16x2_to_float2(pb);
        l[0] += fa.x + fb.x;
        l[1] += fa.y + fb.y;
      }
      // P as the B operand (rows x heads), then O^T += V^T P per 16 dimensions
      const uint32_t b0 = transpose8x8(pa), b1 = transpose8x8(pb);
#pragma unroll
      for (int mb = 0; mb < 2 * NPB; ++mb)
        mma_16816(o[mb], VF[mb][0], VF[mb][1], VF[mb][2], VF[mb][3], b0, b1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == STAGES) {
      s = 0;
      ph ^= 1u;
    }

    if (flags & kLast) {
      if (lane == 0) mbar_arrive(&freeb[buf]);   // done with this item's buffer
      // the warp's state for each head of the group: l summed over the rows
      // (lanes g)
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        l[0] += __shfl_xor_sync(kFull, l[0], o2);
        l[1] += __shfl_xor_sync(kFull, l[1], o2);
      }
      // The warps' states of a head are merged into one before it goes to the
      // workspace, up to four heads a round: every warp writes its states to
      // the merge scratch; once all have (mrg[0]), warp w merges the round's
      // head w and writes it (slot 0); every warp then marks the scratch read
      // (mrg[1]) before the next round or item writes it again.
      float* scr = reinterpret_cast<float*>(smem + C::OFF_MRG);
      bool ok = true;
      for (int r0 = 0; r0 < G; r0 += C::MRGH) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * t + e;
          if (h >= r0 && h < r0 + C::MRGH) {
            // block mb: rows g, g + 8 of O^T are dimensions 16 mb + g, + 8
            float* dst = scr + (warp * C::MRGH + (h - r0)) * (D + 2);
#pragma unroll
            for (int mb = 0; mb < 2 * NPB; ++mb) {
              dst[16 * mb + g] = o[mb][e];
              dst[16 * mb + 8 + g] = o[mb][2 + e];
            }
            if (g == 0) {
              dst[D] = m[e];
              dst[D + 1] = l[e];
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&mrg[0]);
        if (!mbar_wait(&mrg[0], mph, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        if (warp < C::MRGH) {
          const int hr = warp, h = r0 + hr;
          float M = -INFINITY;
#pragma unroll
          for (int i = 0; i < NW; ++i) M = fmaxf(M, scr[(i * C::MRGH + hr) * (D + 2) + D]);
          float L = 0.f, acc[D / 32];
#pragma unroll
          for (int q = 0; q < D / 32; ++q) acc[q] = 0.f;
#pragma unroll
          for (int i = 0; i < NW; ++i) {
            const float* src = scr + (i * C::MRGH + hr) * (D + 2);
            const float mi = src[D];
            const float w = (mi == -INFINITY) ? 0.f : fast_exp2((mi - M) * sl);
            L += w * src[D + 1];
#pragma unroll
            for (int q = 0; q < D / 32; ++q) acc[q] += w * src[lane + 32 * q];
          }
          const size_t ps = ((size_t)(b * p.Hq + h0 + h) * p.nchunk + c) * kPartSlots;
#pragma unroll
          for (int q = 0; q < D / 32; ++q) p.part_acc[ps * D + lane + 32 * q] = acc[q];
          if (lane == 0) *reinterpret_cast<float2*>(p.part_ml + ps * 2) = make_float2(M, L);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&mrg[1]);
        if (!mbar_wait(&mrg[1], mph, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        mph ^= 1u;
      }
      if (!ok) break;
    }
  }
}

template <typename T, int D, int G, int NW, int NP, int TT, int STAGES>
cudaError_t launch_attn_t(const AttnParams& p, int num_sms, cudaStream_t st) {
  using C = AttnCfg<T, D, G, NW, NP, TT, STAGES>;
  auto kfn = attn_kernel<T, D, G, NW, NP, TT, STAGES>;
  static PerDeviceOnce attrs;   // per instantiation and device
  const cudaError_t ea = attrs.run([&]() -> cudaError_t {
    cudaError_t e =
        cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    if (C::RSPLIT) {
      // the register split assumes LREGS registers per thread at launch
      cudaFuncAttributes fa{};
      e = cudaFuncGetAttributes(&fa, kfn);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != C::LREGS) return cudaErrorInvalidConfiguration;
    }
    return cudaSuccess;
  });
  if (ea != cudaSuccess) return ea;
  const int grid = max(1, min(num_sms, p.n_items));
  const cudaError_t e = launch_pdl(kfn, dim3(grid), dim3(C::NT), (size_t)C::SMEM, st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// fp32 caches: 16 warps per CTA, NW consumers and NP producers (builder,
// streaming warps), 4 warps on each SM sub-partition with up to 128 registers
// per thread.
#ifndef LYCHEE_ATTN_NW
#define LYCHEE_ATTN_NW 12
#endif
// tensor-core consumers: far fewer instructions per row, so fewer consumer
// warps and more streaming warps (a builder and seven streaming warps)
#ifndef LYCHEE_ATTN_NW_MMA
#define LYCHEE_ATTN_NW_MMA 4
#endif
#ifndef LYCHEE_ATTN_NP_MMA
#define LYCHEE_ATTN_NP_MMA 8
#endif
#ifndef LYCHEE_ATTN_NP
#define LYCHEE_ATTN_NP 4
#endif
#ifndef LYCHEE_ATTN_RING_KB
#define LYCHEE_ATTN_RING_KB 200
#endif

#ifndef LYCHEE_ATTN_TT
#define LYCHEE_ATTN_TT 128
#endif

// Tile rows: LYCHEE_ATTN_TT rows of up to 256 bytes, half as many of 512 bytes
// (fp32, d = 128).
template <typename T, int D>
constexpr int tile_rows() {
  return D * (int)sizeof(T) > 256 ? LYCHEE_ATTN_TT / 2 : LYCHEE_ATTN_TT;
}

// Ring depth: as many stages (2..8) as the shared memory left by everything else
// holds, within LYCHEE_ATTN_RING_KB of K/V tiles and q.
template <typename T, int D, int G, int NW, int NP, int TT>
constexpr int ring_stages() {
  constexpr int stage = 2 * TT * D * (int)sizeof(T) + (G * D * (int)sizeof(T) + 127) / 128 * 128;
  constexpr int rest = AttnCfg<T, D, G, NW, NP, TT, 1>::SMEM - stage;   // per-stage extras are small
  constexpr int fit = (227 * 1024 - rest) / (stage + 64);
  constexpr int want = (LYCHEE_ATTN_RING_KB * 1024) / stage;
  constexpr int s = fit < want ? fit : want;
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}

template <typename T, int D, int G>
cudaError_t launch_attn_g(const AttnParams& p, int num_sms, cudaStream_t st) {
  constexpr int NW = mma_path<T>() ? LYCHEE_ATTN_NW_MMA : LYCHEE_ATTN_NW;
  constexpr int NP = mma_path<T>() ? LYCHEE_ATTN_NP_MMA : LYCHEE_ATTN_NP;
  constexpr int TT = tile_rows<T, D>();
  constexpr int STAGES = ring_stages<T, D, G, NW, NP, TT>();
  static_assert(AttnCfg<T, D, G, NW, NP, TT, STAGES>::SMEM <= 227 * 1024, "shared memory");
  return launch_attn_t<T, D, G, NW, NP, TT, STAGES>(p, num_sms, st);
}

template <typename T, int D>
cudaError_t launch_attn_d(const AttnParams& p, int G, int num_sms, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn_g<T, D, 1>(p, num_sms, st);
    case 2: return launch_attn_g<T, D, 2>(p, num_sms, st);
    case 4: return launch_attn_g<T, D, 4>(p, num_sms, st);
    case 8: return launch_attn_g<T, D, 8>(p, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int attn_tile_rows(int dtype, int D) {
  if (dtype == 0) return D == 64 ? tile_rows<__nv_bfloat16, 64>() : tile_rows<__nv_bfloat16, 128>();
  return D == 64 ? tile_rows<float, 64>() : tile_rows<float, 128>();
}

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
