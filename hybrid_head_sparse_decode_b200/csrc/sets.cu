// sets.cu -- conversions between the two forms of a key-token set S (method
// steps (3)/(4) of the page "LycheeDecode: Accelerating Long-Context LLM
// Inference via Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541):
// an index row (k_b ascending positions, -1 padded) and a membership bitmap
// (bit j of word w: position 32w + j is in S).  The attention kernel reads sets
// as bitmaps so that the G heads of a KV group can be merged word by word.
#include "blocksel.h"
#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr int kThreads = 256;
constexpr int kEntriesPerCta = 4 * kThreads;   // set entries one build_bits CTA covers

// Index rows of the listed sparse heads -> bitmaps (and, when asked, a bit-exact
// copy of the rows: a sparse head hands its set on unchanged).  Each warp takes
// 32 consecutive entries at a time, loads coalesced along the row.  Every
// bitmap word has exactly one writer, so the row needs no clearing pass and no
// atomics: the lane holding the first entry of a word (the word's leader)
// writes it, with the OR of the word's entries among the warp's 32 (a
// segmented OR over the run of lanes holding that word) and, when the run
// reaches the warp's last lane, of the entries after them; it also writes the
// empty words between the previous entry's word and its own.  A set ends at its
// first -1 (or at the row's k-th entry; the budget k_b does not bound what a
// sparse head reads).  The empty words before the first member and after the
// last one can be thousands; the CTA holding that entry clears them together
// after its entries.  An entry outside [0, n_b), not strictly above its
// predecessor, or after the end of the set sets kErrBadIndex; the row is then
// not a set and its bitmap is unspecified, but every store still stays inside
// the row.
__global__ void __launch_bounds__(kThreads) build_bits_kernel(const __grid_constant__ BuildBitsParams p) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr uint32_t kAllLanes = 0xffffffffu;
  constexpr int kWarps = kThreads / 32;
  // word ranges this CTA clears together: [0] before the first member, [1]
  // after the last (each written by the one thread that finds it)
  __shared__ int s_lo[2], s_hi[2];
  if (threadIdx.x < 2) s_lo[threadIdx.x] = s_hi[threadIdx.x] = 0;
  __syncthreads();
  const int b = blockIdx.x / p.nheads, h = p.heads[blockIdx.x % p.nheads];
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const size_t bh = (size_t)b * p.Hq + h;
  uint32_t* row = p.bitmaps + bh * p.nwords;
  const int words = (n + 31) >> 5;
  const int32_t* idx = p.idx_in + bh * p.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int base = blockIdx.y * kEntriesPerCta;
  constexpr int R = kEntriesPerCta / kThreads;         // chunks of 32 entries per warp
  // every chunk's entries (and the entry before each chunk) loaded up front
  int jr[R], pr[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = base + (r * kWarps + warp) * 32 + lane;
    jr[r] = t < p.k ? idx[t] : -1;
    pr[r] = (lane == 0 && t > 0 && t <= p.k) ? idx[t - 1] : -1;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t0 = base + (r * kWarps + warp) * 32;
    if (t0 >= p.k) break;                              // warp-uniform
    const int t = t0 + lane;
    const bool in = t < p.k;
    const int j = jr[r];
    if (in && p.idx_out) p.idx_out[bh * p.k + t] = j;
    int prev = __shfl_up_sync(kAllLanes, j, 1);
    if (lane == 0) prev = pr[r];
    bool member = false;
    if (in) {
      if (j < 0) {
        // the set ends at its first -1: the words after the last member (all
        // of them for an empty set) are cleared below
        if (t == 0 || prev >= 0) {
          s_lo[1] = t == 0 ? 0 : (prev >> 5) + 1;
          s_hi[1] = words;
        }
      } else if ((t > 0 && prev < 0) || j >= n || j <= prev) {
        flag_error(p.err, kErrBadIndex);   // after the end, out of range, or not ascending
      } else {
        member = true;
      }
    }
    // runs of lanes holding members of one word: a run starts where a lane's
    // key differs from the previous lane's (every non-member has a key of its own)
    const int w = j >> 5;
    const int key = member ? w : -2 - lane;
    const int key_prev = __shfl_up_sync(kAllLanes, key, 1);
    const uint32_t starts = __ballot_sync(kAllLanes, lane == 0 || key != key_prev);
    const uint32_t later = starts & ~((2u << lane) - 1u);   // runs starting after this lane
    const int run_end = later ? __ffs(later) - 1 : 32;      // first lane past this lane's run
    uint32_t bits = member ? 1u << (j & 31) : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(kAllLanes, bits, o);
      if (lane + o < run_end) bits |= y;
    }
    const int j_last = __shfl_sync(kAllLanes, j, 31);
    const int pw = prev >> 5;                          // -1 for the first entry (arithmetic shift)
    if (member && w != pw) {
      if (run_end == 32) {
        // the word's entries may go on past the warp's 32
        int last = j_last;
        for (int u = t0 + 32; u < p.k; ++u) {
          const int ju = idx[u];
          if ((ju >> 5) != w || ju <= last) break;
          bits |= 1u << (ju & 31);
          last = ju;
        }
      }
      row[w] = bits;
      if (pw < 0) {            // the first member: the words before it, below
        s_lo[0] = 0;
        s_hi[0] = w;
      } else {
        for (int g = pw + 1; g < w; ++g) row[g] = 0u;
      }
    }
    if (member && t == p.k - 1) {   // a full row: the words after its last member
      s_lo[1] = w + 1;
      s_hi[1] = words;
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < 2; ++e)
    for (int g = s_lo[e] + threadIdx.x; g < s_hi[e]; g += kThreads) row[g] = 0u;
}

// Bitmaps -> index rows for every head: ascending positions, -1 padded to k.
// A row is cut into parts of kExportWords bitmap words, one CTA per (sequence,
// head, part), one word per thread.  A CTA counts the members before its part
// (the popcounts of the row's earlier words), places its own members by a
// block-wide prefix sum of the words' counts into a shared-memory list (each
// thread writes its word's members), and copies the list to the row with
// consecutive threads on consecutive slots.  The CTA holding the row's last
// word also writes the -1 padding.
constexpr int kExportWords = 256;
__global__ void __launch_bounds__(kExportWords) export_kernel(const __grid_constant__ ExportParams p) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int kWarps = kExportWords / 32;
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t s_before;
  __shared__ int32_t list[kExportWords * 32];
  const int bh = blockIdx.x, b = bh / p.Hq;
  const int n = min(max(p.seqlens[b], 1), p.N_max);
  const int words = (n + 31) >> 5;
  const int w0 = blockIdx.y * kExportWords;
  if (w0 >= words) return;                           // past this sequence's row
  const uint32_t* row = p.bitmaps + (size_t)bh * p.nwords;
  int32_t* out = p.idx + (size_t)bh * p.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t tail = (n & 31) ? ((1u << (n & 31)) - 1u) : 0xffffffffu;
  auto word = [&](int w) -> uint32_t {
    return w < words ? __ldcg(&row[w]) & (w == words - 1 ? tail : 0xffffffffu) : 0u;
  };
  // members in the words before this part
  uint32_t pre = 0;
  for (int w = tid; w < w0; w += kExportWords) pre += __popc(word(w));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, o);
  if (lane == 0) wsum[warp] = pre;
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
    for (int i = 0; i < kWarps; ++i) t += wsum[i];
    s_before = t;
  }
  __syncthreads();
  const uint32_t before = s_before;
  // this thread's word and its members' place in the part
  const int w = w0 + tid;
  uint32_t bits = word(w);
  const uint32_t c = __popc(bits);
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();                                   // wsum is reused
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0, m = 0;
  for (int i = 0; i < kWarps; ++i) {
    wbase += i < warp ? wsum[i] : 0u;
    m += wsum[i];
  }
  uint32_t slot = wbase + incl - c;
  while (bits) {
    const int j = __ffs(bits) - 1;
    bits &= bits - 1u;
    list[slot++] = w * 32 + j;
  }
  __syncthreads();
  for (uint32_t i = tid; i < m; i += kExportWords)
    if (before + i < (uint32_t)p.k) out[before + i] = list[i];
  if (w0 + kExportWords >= words)                    // the row's last part: the padding
    for (int t = (int)(before + m) + tid; t < p.k; t += kExportWords) out[t] = -1;
}

}  // namespace

cudaError_t launch_build_bits(const BuildBitsParams& p, cudaStream_t st) {
  if (p.nheads <= 0) return cudaSuccess;
  // (sequence, head) pairs on x (up to 2^31 - 1), parts of the row on y (up to 65535)
  const dim3 grid((unsigned)(p.B * p.nheads), (unsigned)((p.k + kEntriesPerCta - 1) / kEntriesPerCta));
  const cudaError_t e = launch_pdl(build_bits_kernel, grid, dim3(kThreads), 0, st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_export(const ExportParams& p, cudaStream_t st) {
  const unsigned parts = (unsigned)((p.nwords + kExportWords - 1) / kExportWords);
  const cudaError_t e = launch_pdl(export_kernel, dim3((unsigned)(p.B * p.Hq), parts),
                                   dim3(kExportWords), 0, st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lychee

namespace lychee {
namespace {

// One CTA per (sequence, KV head): the new K and V rows, 16 bytes per thread.
__global__ void __launch_bounds__(64) append_kv_kernel(const __grid_constant__ AppendParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x / p.Hkv;
  const int n = p.seqlens[b];
  if (n < 1 || n > p.N_max) return;
  const size_t unit = blockIdx.x;   // b * Hkv + g
  const int pieces = p.row_bytes / 16;
  const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const char*>(p.k_new) + unit * p.row_bytes);
  const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const char*>(p.v_new) + unit * p.row_bytes);
  uint4* kc = reinterpret_cast<uint4*>(static_cast<char*>(p.k_cache) +
                                       (unit * p.N_max + (size_t)(n - 1)) * p.row_bytes);
  uint4* vc = reinterpret_cast<uint4*>(static_cast<char*>(p.v_cache) +
                                       (unit * p.N_max + (size_t)(n - 1)) * p.row_bytes);
  for (int i = threadIdx.x; i < pieces; i += blockDim.x) {
    kc[i] = kn[i];
    vc[i] = vn[i];
  }
}

}  // namespace

cudaError_t launch_append_kv(const AppendParams& p, cudaStream_t st) {
  const cudaError_t e =
      launch_pdl(append_kv_kernel, dim3((unsigned)(p.B * p.Hkv)), dim3(64), 0, st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lychee
