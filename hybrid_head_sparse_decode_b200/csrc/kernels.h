// kernels.h -- parameter blocks and launchers of the libychee kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lychee {

// Hybrid attention over one layer (attn.cu).
struct AttnParams {
  const void* q;            // [B, Hq, D]
  const void* k;            // [B, Hkv, N_max, D]
  const void* v;            // [B, Hkv, N_max, D]
  const int32_t* seqlens;   // [B]
  const uint32_t* bitmaps;  // [B, Hq, nwords]: incoming sets of sparse heads
  float* logits;            // [B, Hq, N_max]: raw q.k of retrieval heads
  float* part_ml;           // [B, Hq, nchunk, kPartSlots, 2]: (max raw dot, sum of weights)
  float* part_acc;          // [B, Hq, nchunk, kPartSlots, D]: unnormalised weighted values
  int32_t* part_n;          // [B, Hq, nchunk]: partial states written for the chunk
  const int32_t* k_per_seq; // [B] or null (validated here)
  uint32_t* err;
  uint32_t* counter;        // work-item counter, 0 at launch, 0 again at exit
  uint32_t* exits;          // CTAs that finished, 0 at launch, 0 again at exit
  int B, Hq, Hkv, N_max, nwords, nchunk, n_items;
  int chunk;                // positions per work item (multiple of 32, kChunkMin..kChunk)
  int nchunk_run;           // chunks of N_max at that length (<= nchunk, the partials' stride)
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t role[4];         // bit h set: head h is a retrieval head
  int gather_tma;           // 1: sparse rows are gathered through tmk / tmv
  // K and V caches viewed as [B * Hkv * N_max] rows of D elements, box one row
  // (TMA tile::gather4); valid when gather_tma is 1
  alignas(64) CUtensorMap tmk;
  alignas(64) CUtensorMap tmv;
};
cudaError_t launch_attn(const AttnParams& p, int dtype, int D, int G, int num_sms,
                        cudaStream_t st);

// argsTopK of retrieval heads (topk.cu).
struct TopkParams {
  const float* logits;       // [B, Hq, N_max]
  const int32_t* seqlens;    // [B]
  const int32_t* k_per_seq;  // [B] or null
  uint32_t* bitmaps;         // [B, Hq, nwords] or null: selected set as bits
  int32_t* idx_out;          // [B, Hq, k] or null: selected set, ascending, -1 padded
  uint32_t* err;
  int B, Hq, N_max, nwords, k, nheads;
  uint8_t heads[128];        // the retrieval heads handled by this launch
};
cudaError_t launch_topk(const TopkParams& p, cudaStream_t st);

// Merge of split partials into the attention output (combine.cu).
struct CombineParams {
  const float* part_ml;      // [B, Hq, nchunk, kPartSlots, 2]
  const float* part_acc;     // [B, Hq, nchunk, kPartSlots, D]
  const int32_t* part_n;     // [B, Hq, nchunk]: states used per chunk
  const int32_t* seqlens;    // [B]
  void* out;                 // [B, Hq, D]
  uint32_t* err;
  int B, Hq, N_max, nchunk;  // nchunk: the partials' chunk stride
  int chunk;                 // positions per attention work item
  float scale_log2;
};
cudaError_t launch_combine(const CombineParams& p, int dtype, int D, cudaStream_t st);

// The top-k of the retrieval heads and the combine of every head in one launch
// (topk.cu); just the combine when p.nheads is 0.
cudaError_t launch_topk_combine(const TopkParams& p, const CombineParams& cp, int dtype, int D,
                                cudaStream_t st);

// Incoming index sets -> membership bitmaps, with validation; the rows are also
// copied to idx_out (sparse heads pass their set on unchanged) (sets.cu).
struct BuildBitsParams {
  const int32_t* idx_in;     // [B, Hq, k]
  int32_t* idx_out;          // [B, Hq, k] or null
  const int32_t* seqlens;
  const int32_t* k_per_seq;
  uint32_t* bitmaps;         // [B, Hq, nwords]
  uint32_t* err;
  int B, Hq, N_max, nwords, k, nheads;
  uint8_t heads[128];        // the sparse heads whose sets are built
};
cudaError_t launch_build_bits(const BuildBitsParams& p, cudaStream_t st);

// Membership bitmaps -> index rows (ascending, -1 padded) for every head (sets.cu).
struct ExportParams {
  const uint32_t* bitmaps;
  const int32_t* seqlens;
  int32_t* idx;              // [B, Hq, k]
  int B, Hq, N_max, nwords, k;
};
cudaError_t launch_export(const ExportParams& p, cudaStream_t st);

}  // namespace lychee
