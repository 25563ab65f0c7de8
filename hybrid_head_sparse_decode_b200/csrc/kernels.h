// kernels.h -- parameter blocks and launchers of the libychee kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lychee {

// The sliding-window branch of sparse heads, fused into their output by a
// sigmoid gate (combine epilogues; off when k is null).
struct WindowParams {
  const void* q;             // [B, Hq, D]: the layer's queries
  const void* k;             // [B, Hkv, window, D]: window ring (position j in row j % window)
  const void* v;             // [B, Hkv, window, D]
  const float* gate;         // [B, Hq]: gate logits; out = s O_sparse + (1 - s) O_window, s = sigmoid
  int window, Hkv;
  uint32_t role[4];          // bit h set: head h is a retrieval head (no window branch)
};

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
  uint32_t* t_counter;      // tail-combine claim counter, 0 at launch, 0 again at exit
  // Tail: the combine of the previous layer of a stack, run by the CTAs that
  // have no attention item left (t_heads = B * Hq), or none (t_heads = 0).
  const float* t_part_ml;   // the previous layer's partial states (layout of part_ml)
  const float* t_part_acc;
  const int32_t* t_part_n;
  void* t_out;              // [B, Hq, D]: the previous layer's output
  int t_heads;
  WindowParams t_win;       // the previous layer's window branch (t_win.k null: none)
  int B, Hq, Hkv, N_max, nwords, nchunk, n_items;
  int chunk;                // positions per work item (multiple of 32, kChunkMin..kChunk)
  int t_chunk;              // the previous layer's (the chunks of the tail's partial states)
  int nchunk_run;           // chunks of N_max at that length (<= nchunk, the partials' stride)
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t role[4];         // bit h set: head h is a retrieval head
  // Work order: items of the KV groups gorder[0 .. n_indep) come first (their
  // incoming sets are final when the kernel starts), then those of gorder[n_indep
  // .. Hkv), whose sets the previous kernel of the stream may still be writing:
  // the kernel waits for that kernel before it reads them.
  int n_indep;
  uint8_t gorder[128];
  int gather_tma;           // fp32 caches, 1: part of the sparse rows come through tmk / tmv
  unsigned long long wait_ns;  // a pipeline wait gives up (kErrTimeout) after this long
  int withhold_first;       // test only: the builder never announces its first item
  // K and V caches viewed as [B * Hkv * N_max] rows of D elements, box one row
  // (TMA tile::gather4); valid when gather_tma is 1 (fp32 caches)
  alignas(64) CUtensorMap tmk;
  alignas(64) CUtensorMap tmv;
  // bf16 caches (tensor-core consumers): K and V viewed as [B * Hkv][N_max][D],
  // boxes 64 elements wide with a 128-byte swizzle, attn_tile_rows() rows high
  // (*_tile) and 16 rows high (*_rest); the dense tiles come through these
  alignas(64) CUtensorMap tmk_tile;
  alignas(64) CUtensorMap tmk_rest;
  alignas(64) CUtensorMap tmv_tile;
  alignas(64) CUtensorMap tmv_rest;
};
cudaError_t launch_attn(const AttnParams& p, int dtype, int D, int G, int num_sms,
                        cudaStream_t st);
// Rows per shared-memory tile of the attention kernel for this element type and
// head dimension.
int attn_tile_rows(int dtype, int D);

// argsTopK of retrieval heads (topk.cu).
struct TopkParams {
  const float* logits;       // [B, Hq, N_max]
  const int32_t* seqlens;    // [B]
  const int32_t* k_per_seq;  // [B] or null
  uint32_t* bitmaps;         // [B, Hq, nwords] or null: selected set as bits
  int32_t* idx_out;          // [B, Hq, k] or null: selected set, ascending, -1 padded
  uint32_t* err;
  int B, Hq, N_max, nwords, k, nheads;
  int sms;                   // SMs of the device (the cluster size is picked by waves)
  uint8_t heads[128];        // the retrieval heads handled by this launch
};

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
  WindowParams win;          // win.k null: no window branch
};
cudaError_t launch_combine(const CombineParams& p, int dtype, int D, cudaStream_t st);

// The top-k of the retrieval heads and the combine of every head in one launch
// (topk.cu); just the combine when p.nheads is 0, just the top-k when cp.B is 0.
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

// Head roles from HardKuma gate parameters (roles.cu).
struct RolesParams {
  const double* alpha;      // [L, Hq]
  const double* beta;       // [L, Hq]
  uint8_t* role;            // [L, Hq]: 1 retrieval (E[z] > 0.5, or layer 0), 0 sparse
  double* expected_z;       // [L, Hq] or null
  double* expected_l0;      // [1] or null: sum of P(z != 0) over the gated heads
  double p, q;              // stretch limits, p < 0 < 1 < q
  int L, Hq;
  int layer0_retrieval;     // 1: layer 0 is all retrieval and not gated
};
cudaError_t launch_hardkuma_roles(const RolesParams& p, cudaStream_t st);

}  // namespace lychee
