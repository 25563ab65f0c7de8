// blocksel.h -- parameter block and launcher of the block-granular selection
// (blocksel.cu), internal.
#pragma once

#include "kernels.h"

namespace lychee {

// Block-granular selection of retrieval heads' sets (blocksel.cu): blocks of
// `block` positions scored by their largest logit, the max(1, k_b / block) best
// taken whole.  block is a multiple of 32 (whole bitmap words).
struct BlockSelParams {
  const float* logits;       // [B, Hq, N_max]: raw q.k of the retrieval heads
  const int32_t* seqlens;    // [B]
  const int32_t* k_per_seq;  // [B] or null
  uint32_t* bitmaps;         // [B, Hq, nwords] or null
  int32_t* idx_out;          // [B, Hq, k] or null: ascending, -1 padded
  uint32_t* err;
  int B, Hq, N_max, nwords, k, nheads, block;
  uint8_t heads[128];        // the retrieval heads handled by this launch
};
// block keys of one head, at most 32768 blocks (see block_select_smem)
constexpr size_t kBlockSelSmemMax = 16 + (32768 + 32) * 4;
size_t block_select_smem(int N_max, int block);
// The selection of the retrieval heads and the combine of every head in one
// launch; just the combine when p.nheads is 0.
cudaError_t launch_block_select_combine(const BlockSelParams& p, const CombineParams& cp,
                                        int dtype, int D, cudaStream_t st);

// The current token's K and V rows into the caches at row n_b - 1 (sets.cu).
struct AppendParams {
  const void* k_new;         // [B, Hkv, row_bytes]
  const void* v_new;
  void* k_cache;             // [B, Hkv, N_max, row_bytes]
  void* v_cache;
  const int32_t* seqlens;    // [B]
  int B, Hkv, N_max, row_bytes;
};
cudaError_t launch_append_kv(const AppendParams& p, cudaStream_t st);

}  // namespace lychee
