// api.cu -- the C ABI of libychee (declared in include/lychee.h): argument
// validation, workspace layout and the launch sequence of one layer and of an
// L-layer decode step.  Host code only; no memory is allocated here.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "blocksel.h"
#include "kernels.h"
#include "lychee.h"

using namespace lychee;

namespace {

constexpr int kVersion = 100;   // 0.1.0

struct Layout {
  size_t logits, part_ml, part_acc, part_n, bitmaps, total;
  int nchunk, nwords;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

lychee_status check_shape(const lychee_shape* s) {
  if (!s) return LYCHEE_ERR_INVALID_ARG;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->d < 1 || s->N_max < 1 || s->k < 1)
    return LYCHEE_ERR_INVALID_ARG;
  if (s->dtype != LYCHEE_BF16 && s->dtype != LYCHEE_FP32) return LYCHEE_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return LYCHEE_ERR_INVALID_ARG;
  if (s->k > s->N_max) return LYCHEE_ERR_INVALID_ARG;
  const int G = s->Hq / s->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return LYCHEE_ERR_UNSUPPORTED;
  if (s->Hq > kMaxHq) return LYCHEE_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return LYCHEE_ERR_UNSUPPORTED;
  if (s->N_max > (1 << 24)) return LYCHEE_ERR_UNSUPPORTED;
  const long long nchunk = (s->N_max + kChunkMin - 1) / kChunkMin;
  if ((long long)s->B * s->Hkv * nchunk >= (1LL << 31)) return LYCHEE_ERR_UNSUPPORTED;
  if ((long long)s->B * s->Hq >= (1LL << 24)) return LYCHEE_ERR_UNSUPPORTED;
  if (s->block < 0) return LYCHEE_ERR_INVALID_ARG;
  if (s->block > 1) {
    if (s->block % 32 != 0 || s->block > 1024 || s->block > s->k) return LYCHEE_ERR_INVALID_ARG;
    if (block_select_smem(s->N_max, s->block) > kBlockSelSmemMax) return LYCHEE_ERR_UNSUPPORTED;
  }
  return LYCHEE_OK;
}

Layout layout_of(const lychee_shape* s) {
  Layout L{};
  L.nchunk = (s->N_max + kChunkMin - 1) / kChunkMin;   // room for the shortest chunk
  L.nwords = (s->N_max + 31) / 32;
  const size_t bh = (size_t)s->B * s->Hq;
  size_t off = sizeof(WsHeader);
  L.logits = off;
  off += align256(bh * s->N_max * 4);
  L.part_ml = off;
  off += align256(bh * L.nchunk * kPartSlots * 2 * 4);
  L.part_acc = off;
  off += align256(bh * L.nchunk * kPartSlots * s->d * 4);
  L.part_n = off;
  off += align256(bh * L.nchunk * 4);
  L.bitmaps = off;
  off += align256(bh * L.nwords * 4);
  L.total = off;
  return L;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t elem_size(const lychee_shape* s) { return s->dtype == LYCHEE_BF16 ? 2 : 4; }

lychee_status check_roles(const uint8_t* role, int Hq, int* n_sparse) {
  if (!role) return LYCHEE_ERR_INVALID_ARG;
  int ns = 0;
  for (int h = 0; h < Hq; ++h) {
    if (role[h] != LYCHEE_ROLE_SPARSE && role[h] != LYCHEE_ROLE_RETRIEVAL)
      return LYCHEE_ERR_INVALID_ARG;
    ns += role[h] == LYCHEE_ROLE_SPARSE;
  }
  if (n_sparse) *n_sparse = ns;
  return LYCHEE_OK;
}

// ---- device properties -----------------------------------------------------------
int num_sms_current() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> g(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

// ---- tensor maps for the attention kernel's row gathers -----------------------------
// cuTensorMapEncodeTiled comes from the driver through the runtime's entry-point
// query, so the library needs no link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cudaGetLastError();
  });
  return fn;
}

// LYCHEE_NO_TMA_GATHER=1 in the environment (read once) makes every sparse row
// gather use 16-byte copies, the path taken when no tensor map can describe the
// cache; for testing that path.
bool tma_gathers_disabled() {
  static const bool off = [] {
    const char* v = std::getenv("LYCHEE_NO_TMA_GATHER");
    return v && v[0] == '1';
  }();
  return off;
}

// The cache [B, Hkv, N_max, d] as rows of d elements, box one row high and one
// row wide (the form tile::gather4 needs).  False when it cannot be described
// (no encoder, or more rows than a 32-bit coordinate reaches); the kernel then
// gathers with 16-byte copies instead.
bool encode_row_map(CUtensorMap* m, const void* base, const lychee_shape* s) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  const unsigned long long rows = (unsigned long long)s->B * s->Hkv * s->N_max;
  if (!enc || rows > 0x7fffffffull) return false;
  const size_t es = s->dtype == LYCHEE_BF16 ? 2 : 4;
  const cuuint64_t dims[2] = {(cuuint64_t)s->d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)s->d * es};
  const cuuint32_t box[2] = {(cuuint32_t)s->d, 1u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapDataType dt =
      s->dtype == LYCHEE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- optional launch profiler ----------------------------------------------------
struct Profiler {
  std::mutex mu;
  bool on = false;
  int cap = 0, n = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int32_t> kinds;
};
Profiler g_prof;

enum {
  kKindAttn = 0,
  kKindTopk = 1,
  kKindCombine = 2,
  kKindBuildBits = 3,
  kKindExport = 4,
  kKindTopkCombine = 5
};

template <typename F>
cudaError_t timed(int kind, cudaStream_t st, F&& launch) {
  if (!g_prof.on) return launch();
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (!g_prof.on || g_prof.n >= g_prof.cap) return launch();
  const int i = g_prof.n++;
  g_prof.kinds[i] = kind;
  cudaEventRecord(g_prof.ev[2 * i], st);
  const cudaError_t e = launch();
  cudaEventRecord(g_prof.ev[2 * i + 1], st);
  return e;
}

void fill_roles(uint32_t (&bits)[4], const uint8_t* role, int Hq) {
  bits[0] = bits[1] = bits[2] = bits[3] = 0;
  for (int h = 0; h < Hq; ++h)
    if (role[h] == LYCHEE_ROLE_RETRIEVAL) bits[h >> 5] |= 1u << (h & 31);
}

struct Ctx {
  const lychee_shape* s;
  Layout L;
  unsigned char* ws;
  cudaStream_t st;
  int sms;
  WsHeader* hdr() const { return reinterpret_cast<WsHeader*>(ws); }
};

// Positions per attention work item: among the multiples of 32 in
// [kChunkMin, kChunk], the one that minimises the work of the busiest SM for
// full-length sequences, (items per SM, rounded up) x positions per item;
// ties go to the longer chunk (fewer partial states).  Items are claimed
// dynamically, so this only evens out the last wave.
int pick_chunk(const lychee_shape* s, int sms) {
  int best = kChunk;
  long long best_cost = -1;
  for (int cs = kChunk; cs >= kChunkMin; cs -= 32) {
    const long long items = (long long)s->B * s->Hkv * ((s->N_max + cs - 1) / cs);
    const long long cost = (items + sms - 1) / sms * cs;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cs;
    }
  }
  return best;
}

// One layer's launches.  bitmaps carry the sets of sparse heads in and (when
// write_bits) the sets of retrieval heads out.
lychee_status run_layer(const Ctx& c, const void* q, const void* kc, const void* vc,
                        const int32_t* seqlens, const int32_t* k_per_seq, const uint8_t* role,
                        const int32_t* idx_in, void* out, int32_t* idx_out, bool build_bits,
                        bool write_bits) {
  const lychee_shape* s = c.s;
  const int Hq = s->Hq, G = Hq / s->Hkv;
  uint32_t* err = &c.hdr()->err;
  uint32_t* counter = &c.hdr()->counters[0];
  float* logits = reinterpret_cast<float*>(c.ws + c.L.logits);
  float* part_ml = reinterpret_cast<float*>(c.ws + c.L.part_ml);
  float* part_acc = reinterpret_cast<float*>(c.ws + c.L.part_acc);
  int32_t* part_n = reinterpret_cast<int32_t*>(c.ws + c.L.part_n);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(c.ws + c.L.bitmaps);
  uint8_t rheads[kMaxHq], sheads[kMaxHq];
  int nr = 0, ns = 0;
  for (int h = 0; h < Hq; ++h) {
    if (role[h] == LYCHEE_ROLE_RETRIEVAL) rheads[nr++] = (uint8_t)h;
    else sheads[ns++] = (uint8_t)h;
  }
  cudaError_t e = cudaSuccess;
  if (build_bits && ns > 0) {
    BuildBitsParams bp{};
    bp.idx_in = idx_in;
    bp.idx_out = idx_out;
    bp.seqlens = seqlens;
    bp.k_per_seq = k_per_seq;
    bp.bitmaps = bitmaps;
    bp.err = err;
    bp.B = s->B; bp.Hq = Hq; bp.N_max = s->N_max; bp.nwords = c.L.nwords; bp.k = s->k;
    bp.nheads = ns;
    std::memcpy(bp.heads, sheads, ns);
    e = timed(kKindBuildBits, c.st, [&] { return launch_build_bits(bp, c.st); });
    if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
  }
  AttnParams ap{};
  ap.q = q; ap.k = kc; ap.v = vc;
  ap.seqlens = seqlens;
  ap.bitmaps = bitmaps;
  ap.logits = logits;
  ap.part_ml = part_ml;
  ap.part_acc = part_acc;
  ap.part_n = part_n;
  ap.k_per_seq = k_per_seq;
  ap.err = err;
  ap.counter = counter;
  ap.exits = &c.hdr()->counters[1];
  ap.B = s->B; ap.Hq = Hq; ap.Hkv = s->Hkv; ap.N_max = s->N_max;
  ap.nwords = c.L.nwords; ap.nchunk = c.L.nchunk;
  ap.chunk = pick_chunk(s, c.sms);
  ap.nchunk_run = (s->N_max + ap.chunk - 1) / ap.chunk;
  ap.n_items = s->B * s->Hkv * ap.nchunk_run;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s->d));
  fill_roles(ap.role, role, Hq);
  ap.gather_tma = !tma_gathers_disabled() && encode_row_map(&ap.tmk, kc, s) &&
                   encode_row_map(&ap.tmv, vc, s) ? 1 : 0;
  e = timed(kKindAttn, c.st, [&] { return launch_attn(ap, s->dtype, s->d, G, c.sms, c.st); });
  if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
  // top-k of the retrieval heads and the combine of every head: independent
  // (logits vs partial states), so one launch does both
  TopkParams tp{};
  tp.logits = logits;
  tp.seqlens = seqlens;
  tp.k_per_seq = k_per_seq;
  tp.bitmaps = write_bits ? bitmaps : nullptr;
  tp.idx_out = idx_out;
  tp.err = err;
  tp.B = s->B; tp.Hq = Hq; tp.N_max = s->N_max; tp.nwords = c.L.nwords; tp.k = s->k;
  tp.nheads = nr;
  std::memcpy(tp.heads, rheads, nr);
  CombineParams cp{};
  cp.part_ml = part_ml;
  cp.part_acc = part_acc;
  cp.part_n = part_n;
  cp.seqlens = seqlens;
  cp.out = out;
  cp.err = err;
  cp.B = s->B; cp.Hq = Hq; cp.N_max = s->N_max; cp.nchunk = c.L.nchunk;
  cp.chunk = ap.chunk;
  cp.scale_log2 = ap.scale_log2;
  if (s->block > 1 && nr > 0) {
    // block-granular selection and the combine in one launch
    BlockSelParams bp{};
    bp.logits = logits;
    bp.seqlens = seqlens;
    bp.k_per_seq = k_per_seq;
    bp.bitmaps = tp.bitmaps;
    bp.idx_out = tp.idx_out;
    bp.err = err;
    bp.B = s->B; bp.Hq = Hq; bp.N_max = s->N_max; bp.nwords = c.L.nwords; bp.k = s->k;
    bp.nheads = nr;
    bp.block = s->block;
    std::memcpy(bp.heads, rheads, nr);
    e = timed(kKindTopkCombine, c.st,
              [&] { return launch_block_select_combine(bp, cp, s->dtype, s->d, c.st); });
    if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
    return LYCHEE_OK;
  }
  e = timed(nr > 0 ? kKindTopkCombine : kKindCombine, c.st,
            [&] { return launch_topk_combine(tp, cp, s->dtype, s->d, c.st); });
  if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
  return LYCHEE_OK;
}

lychee_status export_sets(const Ctx& c, const int32_t* seqlens, int32_t* idx) {
  ExportParams xp{};
  xp.bitmaps = reinterpret_cast<const uint32_t*>(c.ws + c.L.bitmaps);
  xp.seqlens = seqlens;
  xp.idx = idx;
  xp.B = c.s->B; xp.Hq = c.s->Hq; xp.N_max = c.s->N_max; xp.nwords = c.L.nwords; xp.k = c.s->k;
  const cudaError_t e = timed(kKindExport, c.st, [&] { return launch_export(xp, c.st); });
  return e == cudaSuccess ? LYCHEE_OK : LYCHEE_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t lychee_workspace_size(const lychee_shape* s) {
  if (check_shape(s) != LYCHEE_OK) return 0;
  return layout_of(s).total;
}

lychee_status lychee_workspace_offsets(const lychee_shape* s, size_t* logits_off,
                                      size_t* bitmaps_off, int32_t* nwords) {
  if (check_shape(s) != LYCHEE_OK || !logits_off || !bitmaps_off || !nwords)
    return LYCHEE_ERR_INVALID_ARG;
  const Layout L = layout_of(s);
  *logits_off = L.logits;
  *bitmaps_off = L.bitmaps;
  *nwords = L.nwords;
  return LYCHEE_OK;
}

lychee_status lychee_hybrid_decode_attn(const lychee_shape* s, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* seqlens, const int32_t* k_per_seq,
                                        const uint8_t* head_role, const int32_t* idx_in,
                                        void* out, int32_t* idx_out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  lychee_status st = check_shape(s);
  if (st != LYCHEE_OK) return st;
  int ns = 0;
  if ((st = check_roles(head_role, s->Hq, &ns)) != LYCHEE_OK) return st;
  if (!q || !k_cache || !v_cache || !seqlens || !out || !idx_out) return LYCHEE_ERR_INVALID_ARG;
  if (ns > 0 && !idx_in) return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return LYCHEE_ERR_INVALID_ARG;
  const Layout L = layout_of(s);
  if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256))
    return LYCHEE_ERR_WORKSPACE;
  Ctx c{s, L, static_cast<unsigned char*>(workspace), static_cast<cudaStream_t>(stream), 0};
  if ((c.sms = num_sms_current()) <= 0) return LYCHEE_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, L.logits, c.st) != cudaSuccess) return LYCHEE_ERR_CUDA;
  return run_layer(c, q, k_cache, v_cache, seqlens, k_per_seq, head_role, ns > 0 ? idx_in : nullptr,
                   out, idx_out, /*build_bits=*/true, /*write_bits=*/false);
}

lychee_status lychee_decode_stack(const lychee_shape* s, int32_t L, const void* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seqlens, const int32_t* k_per_seq,
                                  const uint8_t* head_role, void* out, int32_t* idx_final,
                                  int32_t* idx_layers, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  lychee_status st = check_shape(s);
  if (st != LYCHEE_OK) return st;
  if (L < 1 || !q || !k_caches || !v_caches || !seqlens || !head_role || !out || !idx_final)
    return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return LYCHEE_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    if ((st = check_roles(head_role + (size_t)l * s->Hq, s->Hq, nullptr)) != LYCHEE_OK) return st;
    if (!k_caches[l] || !v_caches[l] || !aligned(k_caches[l], 16) || !aligned(v_caches[l], 16))
      return LYCHEE_ERR_INVALID_ARG;
  }
  for (int h = 0; h < s->Hq; ++h)
    if (head_role[h] != LYCHEE_ROLE_RETRIEVAL) return LYCHEE_ERR_INVALID_ARG;
  const Layout lay = layout_of(s);
  if (!workspace || workspace_bytes < lay.total || !aligned(workspace, 256))
    return LYCHEE_ERR_WORKSPACE;
  Ctx c{s, lay, static_cast<unsigned char*>(workspace), static_cast<cudaStream_t>(stream), 0};
  if ((c.sms = num_sms_current()) <= 0) return LYCHEE_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, lay.logits, c.st) != cudaSuccess) return LYCHEE_ERR_CUDA;
  const size_t layer_elems = (size_t)s->B * s->Hq * s->d;
  const size_t esz = elem_size(s);
  for (int l = 0; l < L; ++l) {
    const char* ql = static_cast<const char*>(q) + (size_t)l * layer_elems * esz;
    char* ol = static_cast<char*>(out) + (size_t)l * layer_elems * esz;
    st = run_layer(c, ql, k_caches[l], v_caches[l], seqlens, k_per_seq,
                   head_role + (size_t)l * s->Hq, nullptr, ol, nullptr, /*build_bits=*/false,
                   /*write_bits=*/true);
    if (st != LYCHEE_OK) return st;
    if (idx_layers) {
      st = export_sets(c, seqlens, idx_layers + (size_t)l * s->B * s->Hq * s->k);
      if (st != LYCHEE_OK) return st;
    }
  }
  return export_sets(c, seqlens, idx_final);
}

lychee_status lychee_append_kv(const lychee_shape* s, const void* k_new, const void* v_new,
                               void* k_cache, void* v_cache, const int32_t* seqlens,
                               void* stream) {
  lychee_status st = check_shape(s);
  if (st != LYCHEE_OK) return st;
  if (!k_new || !v_new || !k_cache || !v_cache || !seqlens) return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16))
    return LYCHEE_ERR_INVALID_ARG;
  AppendParams p{};
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.seqlens = seqlens;
  p.B = s->B; p.Hkv = s->Hkv; p.N_max = s->N_max;
  p.row_bytes = s->d * (int)elem_size(s);
  return launch_append_kv(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LYCHEE_OK
                                                                               : LYCHEE_ERR_CUDA;
}

lychee_status lychee_check_device_error(void* workspace, void* stream, uint32_t* detail) {
  if (!workspace) return LYCHEE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LYCHEE_ERR_CUDA;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LYCHEE_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(v)) != cudaSuccess) return LYCHEE_ERR_CUDA;
  if (detail) *detail = v;
  if (v & kErrTimeout) return LYCHEE_ERR_TIMEOUT;
  if (v) return LYCHEE_ERR_BAD_INDEX;
  return LYCHEE_OK;
}

const char* lychee_status_string(lychee_status st) {
  switch (st) {
    case LYCHEE_OK: return "ok";
    case LYCHEE_ERR_INVALID_ARG: return "invalid argument";
    case LYCHEE_ERR_UNSUPPORTED: return "unsupported shape";
    case LYCHEE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LYCHEE_ERR_CUDA: return "CUDA error";
    case LYCHEE_ERR_BAD_INDEX: return "bad incoming index, sequence length or budget";
    case LYCHEE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int32_t lychee_version(void) { return kVersion; }

lychee_status lychee_profile_begin(int32_t max_launches) {
  if (max_launches < 1) return LYCHEE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (g_prof.on) return LYCHEE_ERR_INVALID_ARG;
  if ((int)g_prof.ev.size() < 2 * max_launches) {
    const size_t old = g_prof.ev.size();
    g_prof.ev.resize(2 * (size_t)max_launches);
    for (size_t i = old; i < g_prof.ev.size(); ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
        g_prof.ev.resize(i);
        return LYCHEE_ERR_CUDA;
      }
  }
  g_prof.kinds.assign(max_launches, -1);
  g_prof.cap = max_launches;
  g_prof.n = 0;
  g_prof.on = true;
  return LYCHEE_OK;
}

lychee_status lychee_profile_end(int32_t capacity, int32_t* kinds, float* ms, int32_t* n_out) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (!g_prof.on) return LYCHEE_ERR_INVALID_ARG;
  g_prof.on = false;
  const int n = g_prof.n;
  if (n_out) *n_out = n;
  for (int i = 0; i < n && i < capacity; ++i) {
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return LYCHEE_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess)
      return LYCHEE_ERR_CUDA;
    if (kinds) kinds[i] = g_prof.kinds[i];
    if (ms) ms[i] = t;
  }
  return LYCHEE_OK;
}

}  // extern "C"
