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

// Workspace regions.  The single-layer call uses the first set of logits and
// partial states and ends at `layer_total`; the stack alternates two logits
// regions and three partial-state regions between consecutive layers (layer l
// uses logits l % 2 and partials l % 3), so that a layer's attention can run
// while the previous layer's selection reads its logits and the layer before
// that is still being combined.
constexpr int kLogitBufs = 2;
constexpr int kPartBufs = 3;
struct Layout {
  size_t logits[kLogitBufs], part_ml[kPartBufs], part_acc[kPartBufs], part_n[kPartBufs];
  size_t bitmaps, layer_total, total;
  int nchunk, nwords;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The shortest attention work item the shape may get: kChunkMin positions, or
// kChunkSmall when the layer's K/V rows (B * Hkv * N_max) are too few to give
// every SM an item of kChunkMin.  The partial-state regions hold room for it.
int chunk_lo(const lychee_shape* s) {
  return (long long)s->B * s->Hkv * s->N_max < kSmallLayerRows ? kChunkSmall : kChunkMin;
}

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
  const long long nchunk = (s->N_max + chunk_lo(s) - 1) / chunk_lo(s);
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
  L.nchunk = (s->N_max + chunk_lo(s) - 1) / chunk_lo(s);   // room for the shortest chunk
  L.nwords = (s->N_max + 31) / 32;
  const size_t bh = (size_t)s->B * s->Hq;
  const size_t logits_b = align256(bh * s->N_max * 4);
  const size_t ml_b = align256(bh * L.nchunk * kPartSlots * 2 * 4);
  const size_t acc_b = align256(bh * L.nchunk * kPartSlots * s->d * 4);
  const size_t n_b = align256(bh * L.nchunk * 4);
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += bytes;
    return o;
  };
  // the single-layer call's regions first
  L.logits[0] = take(logits_b);
  L.part_ml[0] = take(ml_b);
  L.part_acc[0] = take(acc_b);
  L.part_n[0] = take(n_b);
  L.bitmaps = take(align256(bh * L.nwords * 4));
  L.layer_total = off;
  for (int i = 1; i < kLogitBufs; ++i) L.logits[i] = take(logits_b);
  for (int i = 1; i < kPartBufs; ++i) {
    L.part_ml[i] = take(ml_b);
    L.part_acc[i] = take(acc_b);
    L.part_n[i] = take(n_b);
  }
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
// gather of fp32 caches use 16-byte copies, the path taken when no tensor map
// can describe the cache; for testing that path.
bool tma_gathers_disabled() {
  static const bool off = [] {
    const char* v = std::getenv("LYCHEE_NO_TMA_GATHER");
    return v && v[0] == '1';
  }();
  return off;
}

// Failure-path testing of the attention kernel's bounded waits, read once from
// the environment: LYCHEE_TEST_WAIT_LIMIT_MS=<ms> shortens the limit after
// which its pipeline waits give up (default 2 s), and
// LYCHEE_TEST_WITHHOLD_ITEM=1 makes every CTA's builder withhold the
// announcement of its first work item, so that the waits on that item run out:
// the call then reports LYCHEE_ERR_TIMEOUT through lychee_check_device_error
// and every kernel returns.  Neither is meant for use outside tests.
uint64_t attn_wait_limit_ns() {
  static const uint64_t ns = [] {
    const char* v = std::getenv("LYCHEE_TEST_WAIT_LIMIT_MS");
    const long ms = v ? std::strtol(v, nullptr, 10) : 0;
    return ms > 0 ? (uint64_t)ms * 1000000ull : kWaitLimitNs;
  }();
  return ns;
}
bool attn_withhold_first_item() {
  static const bool on = [] {
    const char* v = std::getenv("LYCHEE_TEST_WITHHOLD_ITEM");
    return v && v[0] == '1';
  }();
  return on;
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

// bf16 K or V cache [B, Hkv, N_max, d] as a 3-D tensor (d, N_max, B * Hkv),
// boxes 64 elements wide and `rows` high with a 128-byte swizzle: the form in
// which the attention kernel's tensor-core consumers take dense tiles.  Rows
// past N_max read as zero.  False when the driver offers no encoder or refuses
// the map.
bool encode_tile_map(CUtensorMap* m, const void* base, const lychee_shape* s, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)s->d, (cuuint64_t)s->N_max,
                              (cuuint64_t)s->B * (cuuint64_t)s->Hkv};
  const cuuint64_t strides[2] = {(cuuint64_t)s->d * 2, (cuuint64_t)s->N_max * s->d * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- optional launch profiler ----------------------------------------------------
// Per-launch mode: two events around every launch.  Span mode: two events per
// stack call, before its first attention launch and after its last one, and
// none in between, so that the layers still overlap.
struct Profiler {
  std::mutex mu;
  bool on = false;
  bool spans = false;
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
  kKindTopkCombine = 5,
  kKindAttnSpan = 6
};

// Span mode: open (end = false) or close (end = true) the current stack call's
// attention span on `st`.
void span_mark(bool end, cudaStream_t st) {
  if (!g_prof.on || !g_prof.spans) return;
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (!g_prof.on || !g_prof.spans) return;
  if (!end) {
    if (g_prof.n >= g_prof.cap) return;
    const int i = g_prof.n++;
    g_prof.kinds[i] = -1;   // open
    cudaEventRecord(g_prof.ev[2 * i], st);
  } else if (g_prof.n > 0 && g_prof.kinds[g_prof.n - 1] == -1) {
    const int i = g_prof.n - 1;
    g_prof.kinds[i] = kKindAttnSpan;
    cudaEventRecord(g_prof.ev[2 * i + 1], st);
  }
}

template <typename F>
cudaError_t timed(int kind, cudaStream_t st, F&& launch) {
  if (!g_prof.on || g_prof.spans) return launch();
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (!g_prof.on || g_prof.spans || g_prof.n >= g_prof.cap) return launch();
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

// Positions per attention work item, a multiple of 32 in [chunk_lo(s), kChunk].
// A single layer: the one that minimises the work of the busiest SM for
// full-length sequences, (items per SM, rounded up) x positions per item; ties
// go to the longer chunk (fewer partial states).  Items are claimed
// dynamically, so this only evens out the last wave (and, for a small layer,
// spreads its rows over more SMs).  A stack's middle layer (`overlapped`): the
// next layer's CTAs take the SMs this one's last wave leaves, so the longest
// chunk that still gives every SM an item (fewer items: fewer item ends and
// partial states; measured at 128K, 960 positions against 896: 20 us less per
// step).
int pick_chunk(const lychee_shape* s, int sms, bool overlapped) {
  if (overlapped) {
    for (int cs = kChunk; cs >= chunk_lo(s); cs -= 32)
      if ((long long)s->B * s->Hkv * ((s->N_max + cs - 1) / cs) >= sms) return cs;
  }
  int best = kChunk;
  long long best_cost = -1;
  for (int cs = kChunk; cs >= chunk_lo(s); cs -= 32) {
    const long long items = (long long)s->B * s->Hkv * ((s->N_max + cs - 1) / cs);
    const long long cost = (items + sms - 1) / sms * cs;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cs;
    }
  }
  return best;
}

// How one layer's launches are placed in a call.
struct LayerPlan {
  int lbuf = 0, pbuf = 0;      // logits / partial-state regions of this layer
  bool build_bits = false;     // single layer: incoming index rows -> bitmaps first
  bool write_bits = false;     // stack: the retrieval heads' sets go to the bitmaps
  bool fused_combine = true;   // the combine shares the selection launch (single layer,
                               // a stack's last layer)
  const uint8_t* prev_role = nullptr;   // stack: the previous layer's roles (null: none)
  int tail_pbuf = -1;          // stack: partial region of the previous layer, combined
  void* tail_out = nullptr;    //   by this layer's attention CTAs into tail_out
  int chunk = 0;               // positions per work item (0: the single-layer rule)
  int tail_chunk = 0;          // stack: the previous layer's
  bool span_start = false;     // profiler span mode: the stack's first / last
  bool span_end = false;       //   attention launch
  WindowParams win{};          // this layer's window branch, combined with fused_combine
                               // (k null: none)
  WindowParams tail_win{};     // the previous layer's window branch (stack)
};

// The window branch of one layer: its ring caches, gate logits and roles.
WindowParams window_of(const lychee_shape* s, const void* q, const void* k, const void* v,
                       int window, const float* gate, const uint8_t* role) {
  WindowParams w{};
  if (!k) return w;
  w.q = q;
  w.k = k;
  w.v = v;
  w.gate = gate;
  w.window = window;
  w.Hkv = s->Hkv;
  fill_roles(w.role, role, s->Hq);
  return w;
}

// Host checks of a window branch's arguments (k non-null means "on").
lychee_status check_window(const void* k, const void* v, int window, const float* gate) {
  if (!k) return LYCHEE_OK;
  if (!v || !gate || window < 1 || window > kMaxWindow) return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(gate, 4)) return LYCHEE_ERR_INVALID_ARG;
  return LYCHEE_OK;
}

// KV groups in the order the attention kernel takes them: first the groups
// whose sparse heads' sets are final when the kernel starts, then the groups
// holding a sparse head whose set the previous layer's selection is still
// writing (its head was a retrieval head there).  Returns the count of the first.
int group_order(const uint8_t* role, const uint8_t* prev_role, int Hq, int Hkv, uint8_t* order) {
  const int G = Hq / Hkv;
  int n = 0;
  auto dependent = [&](int g) {
    if (!prev_role) return false;
    for (int t = 0; t < G; ++t) {
      const int h = g * G + t;
      if (role[h] == LYCHEE_ROLE_SPARSE && prev_role[h] == LYCHEE_ROLE_RETRIEVAL) return true;
    }
    return false;
  };
  for (int g = 0; g < Hkv; ++g)
    if (!dependent(g)) order[n++] = (uint8_t)g;
  const int n_indep = n;
  for (int g = 0; g < Hkv; ++g)
    if (dependent(g)) order[n++] = (uint8_t)g;
  return n_indep;
}

// One layer's launches.  bitmaps carry the sets of sparse heads in and (when
// plan.write_bits) the sets of retrieval heads out.  The single-layer call
// (build_bits, fused_combine) waits for the previous kernel before the first
// work item; in a stack the attention kernel starts on the groups whose sets
// are final while the previous layer's selection still runs and combines the
// layer before in its tail; only the last layer's selection launch holds a
// combine.
lychee_status run_layer(const Ctx& c, const void* q, const void* kc, const void* vc,
                        const int32_t* seqlens, const int32_t* k_per_seq, const uint8_t* role,
                        const int32_t* idx_in, void* out, int32_t* idx_out,
                        const LayerPlan& plan) {
  const lychee_shape* s = c.s;
  const int Hq = s->Hq, G = Hq / s->Hkv;
  uint32_t* err = &c.hdr()->err;
  // work / exit / tail counters of the attention launch, alternating by layer
  uint32_t* ctr = &c.hdr()->counters[4 * (plan.lbuf & 1)];
  float* logits = reinterpret_cast<float*>(c.ws + c.L.logits[plan.lbuf]);
  float* part_ml = reinterpret_cast<float*>(c.ws + c.L.part_ml[plan.pbuf]);
  float* part_acc = reinterpret_cast<float*>(c.ws + c.L.part_acc[plan.pbuf]);
  int32_t* part_n = reinterpret_cast<int32_t*>(c.ws + c.L.part_n[plan.pbuf]);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(c.ws + c.L.bitmaps);
  uint8_t rheads[kMaxHq], sheads[kMaxHq];
  int nr = 0, ns = 0;
  for (int h = 0; h < Hq; ++h) {
    if (role[h] == LYCHEE_ROLE_RETRIEVAL) rheads[nr++] = (uint8_t)h;
    else sheads[ns++] = (uint8_t)h;
  }
  // the cache's tensor maps first: a map the driver refuses fails the call
  // before anything of the layer is launched
  AttnParams ap{};
  if (s->dtype == LYCHEE_BF16) {
    // dense K / V tiles through swizzled boxes (sparse rows: 16-byte copies)
    const int tt = attn_tile_rows(s->dtype, s->d);
    if (!(encode_tile_map(&ap.tmk_tile, kc, s, tt) && encode_tile_map(&ap.tmk_rest, kc, s, 16) &&
          encode_tile_map(&ap.tmv_tile, vc, s, tt) && encode_tile_map(&ap.tmv_rest, vc, s, 16)))
      return LYCHEE_ERR_CUDA;
  } else {
    ap.gather_tma = !tma_gathers_disabled() && encode_row_map(&ap.tmk, kc, s) &&
                     encode_row_map(&ap.tmv, vc, s) ? 1 : 0;
  }
  cudaError_t e = cudaSuccess;
  if (plan.build_bits && ns > 0) {
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
  ap.q = q; ap.k = kc; ap.v = vc;
  ap.seqlens = seqlens;
  ap.bitmaps = bitmaps;
  ap.logits = logits;
  ap.part_ml = part_ml;
  ap.part_acc = part_acc;
  ap.part_n = part_n;
  ap.k_per_seq = k_per_seq;
  ap.err = err;
  ap.counter = ctr;
  ap.exits = ctr + 1;
  ap.t_counter = ctr + 2;
  ap.B = s->B; ap.Hq = Hq; ap.Hkv = s->Hkv; ap.N_max = s->N_max;
  ap.nwords = c.L.nwords; ap.nchunk = c.L.nchunk;
  ap.chunk = plan.chunk > 0 ? plan.chunk : pick_chunk(s, c.sms, false);
  ap.nchunk_run = (s->N_max + ap.chunk - 1) / ap.chunk;
  ap.n_items = s->B * s->Hkv * ap.nchunk_run;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s->d));
  fill_roles(ap.role, role, Hq);
  if (plan.build_bits) {
    // every group waits: the bitmaps come from the launch just before
    for (int g = 0; g < s->Hkv; ++g) ap.gorder[g] = (uint8_t)g;
    ap.n_indep = 0;
  } else {
    ap.n_indep = group_order(role, plan.prev_role, Hq, s->Hkv, ap.gorder);
  }
  if (plan.tail_pbuf >= 0) {
    ap.t_part_ml = reinterpret_cast<const float*>(c.ws + c.L.part_ml[plan.tail_pbuf]);
    ap.t_part_acc = reinterpret_cast<const float*>(c.ws + c.L.part_acc[plan.tail_pbuf]);
    ap.t_part_n = reinterpret_cast<const int32_t*>(c.ws + c.L.part_n[plan.tail_pbuf]);
    ap.t_out = plan.tail_out;
    ap.t_chunk = plan.tail_chunk;
    ap.t_heads = s->B * Hq;
    ap.t_win = plan.tail_win;
  }
  ap.wait_ns = attn_wait_limit_ns();
  ap.withhold_first = attn_withhold_first_item() ? 1 : 0;
  if (plan.span_start) span_mark(false, c.st);
  e = timed(kKindAttn, c.st, [&] { return launch_attn(ap, s->dtype, s->d, G, c.sms, c.st); });
  if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
  if (plan.span_end) span_mark(true, c.st);
  // the retrieval heads' selection; in the single-layer call the same launch
  // combines every head (logits vs partial states: disjoint inputs and outputs)
  TopkParams tp{};
  tp.logits = logits;
  tp.seqlens = seqlens;
  tp.k_per_seq = k_per_seq;
  tp.bitmaps = plan.write_bits ? bitmaps : nullptr;
  tp.idx_out = idx_out;
  tp.err = err;
  tp.B = s->B; tp.Hq = Hq; tp.N_max = s->N_max; tp.nwords = c.L.nwords; tp.k = s->k;
  tp.nheads = nr;
  tp.sms = c.sms;
  std::memcpy(tp.heads, rheads, nr);
  CombineParams cp{};
  cp.part_ml = part_ml;
  cp.part_acc = part_acc;
  cp.part_n = part_n;
  cp.seqlens = seqlens;
  cp.out = out;
  cp.err = err;
  cp.B = plan.fused_combine ? s->B : 0;   // B = 0: no combine CTAs
  cp.Hq = Hq; cp.N_max = s->N_max; cp.nchunk = c.L.nchunk;
  cp.chunk = ap.chunk;
  cp.scale_log2 = ap.scale_log2;
  cp.win = plan.win;
  if (nr == 0 && !plan.fused_combine) return LYCHEE_OK;
  if (s->block > 1 && nr > 0) {
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
    e = timed(plan.fused_combine ? kKindTopkCombine : kKindTopk, c.st,
              [&] { return launch_block_select_combine(bp, cp, s->dtype, s->d, c.st); });
    if (e != cudaSuccess) return LYCHEE_ERR_CUDA;
    return LYCHEE_OK;
  }
  e = timed(nr == 0 ? kKindCombine : (plan.fused_combine ? kKindTopkCombine : kKindTopk), c.st,
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

size_t lychee_layer_workspace_size(const lychee_shape* s) {
  if (check_shape(s) != LYCHEE_OK) return 0;
  return layout_of(s).layer_total;
}

lychee_status lychee_workspace_offsets(const lychee_shape* s, size_t* logits_off,
                                      size_t* bitmaps_off, int32_t* nwords) {
  if (check_shape(s) != LYCHEE_OK || !logits_off || !bitmaps_off || !nwords)
    return LYCHEE_ERR_INVALID_ARG;
  const Layout L = layout_of(s);
  *logits_off = L.logits[0];
  *bitmaps_off = L.bitmaps;
  *nwords = L.nwords;
  return LYCHEE_OK;
}

}  // extern "C"

namespace {

lychee_status layer_impl(const lychee_shape* s, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* seqlens, const int32_t* k_per_seq,
                         const uint8_t* head_role, const int32_t* idx_in, const void* swa_k,
                         const void* swa_v, int32_t window, const float* gate, void* out,
                         int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream) {
  lychee_status st = check_shape(s);
  if (st != LYCHEE_OK) return st;
  int ns = 0;
  if ((st = check_roles(head_role, s->Hq, &ns)) != LYCHEE_OK) return st;
  if (!q || !k_cache || !v_cache || !seqlens || !out || !idx_out) return LYCHEE_ERR_INVALID_ARG;
  if (ns > 0 && !idx_in) return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return LYCHEE_ERR_INVALID_ARG;
  if ((st = check_window(swa_k, swa_v, window, gate)) != LYCHEE_OK) return st;
  const Layout L = layout_of(s);
  if (!workspace || workspace_bytes < L.layer_total || !aligned(workspace, 256))
    return LYCHEE_ERR_WORKSPACE;
  Ctx c{s, L, static_cast<unsigned char*>(workspace), static_cast<cudaStream_t>(stream), 0};
  if ((c.sms = num_sms_current()) <= 0) return LYCHEE_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), c.st) != cudaSuccess) return LYCHEE_ERR_CUDA;
  LayerPlan plan;
  plan.build_bits = true;
  plan.win = window_of(s, q, swa_k, swa_v, window, gate, head_role);
  return run_layer(c, q, k_cache, v_cache, seqlens, k_per_seq, head_role, ns > 0 ? idx_in : nullptr,
                   out, idx_out, plan);
}

lychee_status stack_impl(const lychee_shape* s, int32_t L, const void* q,
                         const void* const* k_caches, const void* const* v_caches,
                         const int32_t* seqlens, const int32_t* k_per_seq,
                         const uint8_t* head_role, const void* const* swa_k,
                         const void* const* swa_v, int32_t window, const float* gate, void* out,
                         int32_t* idx_final, int32_t* idx_layers, void* workspace,
                         size_t workspace_bytes, void* stream) {
  lychee_status st = check_shape(s);
  if (st != LYCHEE_OK) return st;
  if (L < 1 || !q || !k_caches || !v_caches || !seqlens || !head_role || !out || !idx_final)
    return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return LYCHEE_ERR_INVALID_ARG;
  if (swa_k && (!swa_v || !gate)) return LYCHEE_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    if ((st = check_roles(head_role + (size_t)l * s->Hq, s->Hq, nullptr)) != LYCHEE_OK) return st;
    if (!k_caches[l] || !v_caches[l] || !aligned(k_caches[l], 16) || !aligned(v_caches[l], 16))
      return LYCHEE_ERR_INVALID_ARG;
    if (swa_k) {
      if (!swa_k[l] || !swa_v[l]) return LYCHEE_ERR_INVALID_ARG;
      if ((st = check_window(swa_k[l], swa_v[l], window, gate)) != LYCHEE_OK) return st;
    }
  }
  for (int h = 0; h < s->Hq; ++h)
    if (head_role[h] != LYCHEE_ROLE_RETRIEVAL) return LYCHEE_ERR_INVALID_ARG;
  const Layout lay = layout_of(s);
  if (!workspace || workspace_bytes < lay.total || !aligned(workspace, 256))
    return LYCHEE_ERR_WORKSPACE;
  Ctx c{s, lay, static_cast<unsigned char*>(workspace), static_cast<cudaStream_t>(stream), 0};
  if ((c.sms = num_sms_current()) <= 0) return LYCHEE_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), c.st) != cudaSuccess) return LYCHEE_ERR_CUDA;
  const size_t layer_elems = (size_t)s->B * s->Hq * s->d;
  const size_t esz = elem_size(s);
  auto q_of = [&](int l) { return static_cast<const char*>(q) + (size_t)l * layer_elems * esz; };
  auto out_of = [&](int l) { return static_cast<char*>(out) + (size_t)l * layer_elems * esz; };
  auto win_of = [&](int l) {
    return swa_k ? window_of(s, q_of(l), swa_k[l], swa_v[l], window,
                             gate + (size_t)l * s->B * s->Hq, head_role + (size_t)l * s->Hq)
                 : WindowParams{};
  };
  // Work-item length per layer: a middle layer's last wave is overlapped by the
  // next layer's attention, so it takes the longest items; layer 0 (whose
  // successor waits for all of its sets) and the last layer (whose combine
  // waits for it) take the single-layer rule, which evens out the last wave.
  auto chunk_of = [&](int l) { return pick_chunk(s, c.sms, l > 0 && l < L - 1); };
  for (int l = 0; l < L; ++l) {
    LayerPlan plan;
    plan.chunk = chunk_of(l);
    if (l > 0) plan.tail_chunk = chunk_of(l - 1);
    plan.lbuf = l % kLogitBufs;
    plan.pbuf = l % kPartBufs;
    plan.write_bits = true;
    // every layer but the last is combined by the next layer's attention; the
    // last one's combine shares its selection launch
    plan.fused_combine = l == L - 1;
    if (plan.fused_combine) plan.win = win_of(l);
    plan.span_start = l == 0;
    plan.span_end = l == L - 1;
    if (l > 0) {
      plan.prev_role = head_role + (size_t)(l - 1) * s->Hq;
      plan.tail_pbuf = (l - 1) % kPartBufs;
      plan.tail_out = out_of(l - 1);
      plan.tail_win = win_of(l - 1);
    }
    st = run_layer(c, q_of(l), k_caches[l], v_caches[l], seqlens, k_per_seq,
                   head_role + (size_t)l * s->Hq, nullptr, plan.fused_combine ? out_of(l) : nullptr,
                   nullptr, plan);
    if (st != LYCHEE_OK) return st;
    if (idx_layers) {
      st = export_sets(c, seqlens, idx_layers + (size_t)l * s->B * s->Hq * s->k);
      if (st != LYCHEE_OK) return st;
    }
  }
  return export_sets(c, seqlens, idx_final);
}

}  // namespace

extern "C" {

lychee_status lychee_hybrid_decode_attn(const lychee_shape* s, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* seqlens, const int32_t* k_per_seq,
                                        const uint8_t* head_role, const int32_t* idx_in,
                                        void* out, int32_t* idx_out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  return layer_impl(s, q, k_cache, v_cache, seqlens, k_per_seq, head_role, idx_in, nullptr,
                    nullptr, 0, nullptr, out, idx_out, workspace, workspace_bytes, stream);
}

lychee_status lychee_hybrid_decode_attn_swa(const lychee_shape* s, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* seqlens, const int32_t* k_per_seq,
                                            const uint8_t* head_role, const int32_t* idx_in,
                                            const void* swa_k, const void* swa_v, int32_t window,
                                            const float* gate, void* out, int32_t* idx_out,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  if (!swa_k) return LYCHEE_ERR_INVALID_ARG;
  return layer_impl(s, q, k_cache, v_cache, seqlens, k_per_seq, head_role, idx_in, swa_k, swa_v,
                    window, gate, out, idx_out, workspace, workspace_bytes, stream);
}

lychee_status lychee_decode_stack(const lychee_shape* s, int32_t L, const void* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seqlens, const int32_t* k_per_seq,
                                  const uint8_t* head_role, void* out, int32_t* idx_final,
                                  int32_t* idx_layers, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return stack_impl(s, L, q, k_caches, v_caches, seqlens, k_per_seq, head_role, nullptr, nullptr,
                    0, nullptr, out, idx_final, idx_layers, workspace, workspace_bytes, stream);
}

lychee_status lychee_decode_stack_swa(const lychee_shape* s, int32_t L, const void* q,
                                      const void* const* k_caches, const void* const* v_caches,
                                      const int32_t* seqlens, const int32_t* k_per_seq,
                                      const uint8_t* head_role, const void* const* swa_k,
                                      const void* const* swa_v, int32_t window, const float* gate,
                                      void* out, int32_t* idx_final, int32_t* idx_layers,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!swa_k) return LYCHEE_ERR_INVALID_ARG;
  return stack_impl(s, L, q, k_caches, v_caches, seqlens, k_per_seq, head_role, swa_k, swa_v,
                    window, gate, out, idx_final, idx_layers, workspace, workspace_bytes, stream);
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

lychee_status lychee_hardkuma_roles(const double* alpha, const double* beta, int32_t L,
                                    int32_t Hq, double p, double q, int32_t layer0_retrieval,
                                    uint8_t* head_role, double* expected_z, double* expected_l0,
                                    void* stream) {
  if (!alpha || !beta || !head_role || L < 1 || Hq < 1) return LYCHEE_ERR_INVALID_ARG;
  if ((long long)L * Hq >= (1LL << 31)) return LYCHEE_ERR_UNSUPPORTED;
  if (!(p < 0.0) || !(q > 1.0) || !std::isfinite(p) || !std::isfinite(q))
    return LYCHEE_ERR_INVALID_ARG;
  if (!aligned(alpha, 8) || !aligned(beta, 8) || !aligned(expected_z, 8) ||
      !aligned(expected_l0, 8))
    return LYCHEE_ERR_INVALID_ARG;
  RolesParams rp{};
  rp.alpha = alpha;
  rp.beta = beta;
  rp.role = head_role;
  rp.expected_z = expected_z;
  rp.expected_l0 = expected_l0;
  rp.p = p;
  rp.q = q;
  rp.L = L;
  rp.Hq = Hq;
  rp.layer0_retrieval = layer0_retrieval ? 1 : 0;
  return launch_hardkuma_roles(rp, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LYCHEE_OK
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

}  // extern "C"

namespace {

lychee_status profile_begin(int32_t max_records, bool spans) {
  if (max_records < 1) return LYCHEE_ERR_INVALID_ARG;
  const int32_t max_launches = max_records;
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
  g_prof.spans = spans;
  g_prof.on = true;
  return LYCHEE_OK;
}

}  // namespace

extern "C" {

lychee_status lychee_profile_begin(int32_t max_launches) {
  return profile_begin(max_launches, false);
}

lychee_status lychee_profile_spans_begin(int32_t max_spans) {
  return profile_begin(max_spans, true);
}

lychee_status lychee_profile_end(int32_t capacity, int32_t* kinds, float* ms, int32_t* n_out) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (!g_prof.on) return LYCHEE_ERR_INVALID_ARG;
  g_prof.on = false;
  int n = g_prof.n;
  if (n > 0 && g_prof.kinds[n - 1] == -1) --n;   // a span left open (a failed call)
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
