/*
 * lychee.h -- C ABI of libychee, a B200 (sm_100a) implementation of the
 * hybrid-head sparse decode-attention step of LycheeDecode.
 *
 * The operation (page "LycheeDecode: Accelerating Long-Context LLM Inference
 * via Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541, method
 * steps (1), (3), (4), (7)): at one new token, for every layer,
 *   - a retrieval head h computes s_j = q_h . K_{g,j} / sqrt(d) over every
 *     position j < n_b of its KV group g, O_h = softmax(s) V_g, and hands
 *     S' = argsTopK(s, k_b) to the head at the same index h of the next layer;
 *   - a sparse head h computes O_h = softmax(q_h . K_{g,S}^T / sqrt(d)) V_{g,S}
 *     over its incoming set S only and hands S on unchanged;
 *   - layer 0 is all retrieval (step (1)); roles are fixed inputs (step (7)).
 * The budget k_b = 30% of the sequence length comes from the same page's
 * reproduction paragraph; the caller passes it.
 *
 * Conventions shared by every entry point
 *   - GQA: query head h reads KV head g = h / G with G = Hq / Hkv (consecutive
 *     query heads share a KV head).
 *   - Index sets are int32 rows of capacity k: the first k_b entries are the
 *     set in strictly ascending position order, the rest are -1.
 *     k_b = min(k_per_seq[b] (or k when k_per_seq is NULL), k, n_b).
 *   - argsTopK ranks positions by larger logit first and, on equal logits, by
 *     lower position; the returned set is in ascending position order.
 *   - Element types: LYCHEE_BF16 (16-bit bfloat16) or LYCHEE_FP32.  With fp32
 *     caches all arithmetic is fp32.  With bf16 caches the products q.K and
 *     p.V run on the tensor cores with bf16 operands and fp32 accumulation:
 *     the logits are exact bf16 products summed in fp32, and the softmax
 *     weights p are rounded to bf16 for p.V, with the normaliser summing the
 *     same rounded weights.  Softmax, top-k and combine are fp32.  Outputs are
 *     rounded to the input type (round to nearest even).
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     memory, never synchronises inside a call, and launches only on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream), so a call can be
 *     captured into a CUDA graph.  Calls sharing one workspace must be ordered
 *     on the same stream.
 *   - Errors found on the host (NULL pointers, unsupported shapes, short
 *     workspace, misaligned pointers, a sparse role in layer 0 of a stack) are
 *     returned before anything is launched.  Errors only visible on the device
 *     (an incoming index out of range or not strictly ascending, a sequence
 *     length outside [1, N_max], a budget below 1, a wait that gave up) never
 *     trap: the offending entry is skipped or clamped, a flag is set in the
 *     workspace, and lychee_check_device_error() reports it.
 *   - Device pointers must be 16-byte aligned (q, caches, out, workspace).
 *     bf16 K and V caches are also described to the driver as TMA tensor maps
 *     (cuTensorMapEncodeTiled) before the attention launch; if the driver
 *     offers no encoder or refuses the map, the call returns LYCHEE_ERR_CUDA
 *     with nothing of that layer launched.
 *   - Threads and devices: every call launches on the current device (the
 *     pointers it is given must live there).  The first call of each kernel
 *     configuration on a device sets that kernel's attributes (dynamic shared
 *     memory, cluster size) there and records it per device (atomically, for
 *     device ordinals below 64; higher ordinals set them on every call), so
 *     calls on several devices and from several host threads are fine as long
 *     as calls sharing a workspace are ordered on one stream.
 */
#ifndef LYCHEE_H
#define LYCHEE_H

#include <stddef.h>
#include <stdint.h>

#if defined(LYCHEE_BUILD) && defined(__GNUC__)
#define LYCHEE_API __attribute__((visibility("default")))
#else
#define LYCHEE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LYCHEE_OK = 0,
  LYCHEE_ERR_INVALID_ARG = 1, /* NULL pointer, bad shape, bad role value, misalignment */
  LYCHEE_ERR_UNSUPPORTED = 2, /* shape outside what the kernels are built for      */
  LYCHEE_ERR_WORKSPACE = 3,   /* workspace NULL, misaligned or too small for the call */
  LYCHEE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed               */
  LYCHEE_ERR_BAD_INDEX = 5,   /* device-side: bad incoming index / length / budget  */
  LYCHEE_ERR_TIMEOUT = 6      /* device-side: a pipeline wait gave up (never expected) */
} lychee_status;

typedef enum { LYCHEE_BF16 = 0, LYCHEE_FP32 = 1 } lychee_dtype;

enum { LYCHEE_ROLE_SPARSE = 0, LYCHEE_ROLE_RETRIEVAL = 1 };

/* Problem shape.  Supported: Hq % Hkv == 0 with G = Hq / Hkv in {1, 2, 4, 8},
 * Hq <= 128, d in {64, 128}, 1 <= k <= N_max <= 2^24, B >= 1.
 *
 * block selects how a retrieval head picks the set it hands on (method step
 * (3)): 0 or 1, argsTopK of its logits (k_b positions); a multiple of 32 in
 * [32, 1024] with block <= k and ceil(N_max / block) <= 32768, block-granular
 * selection: the positions are cut into blocks of `block` (the last one
 * shorter), a block's score is its largest logit, and the max(1, floor(k_b /
 * block)) best blocks (ties: lower block index) are taken whole -- the
 * block-sparse reading of the page's decoding kernel, with the block-level
 * maximum scores and k/B top blocks of the HySparse page (B = 64).  A set
 * then holds up to k_b positions (at least one block) and its index row ends
 * at the first -1. */
typedef struct {
  int32_t B;      /* batch (sequences)                         */
  int32_t Hq;     /* query heads                               */
  int32_t Hkv;    /* key/value heads                           */
  int32_t d;      /* head dimension                            */
  int32_t N_max;  /* cache capacity in positions               */
  int32_t dtype;  /* lychee_dtype of q, caches and out         */
  int32_t k;      /* capacity of an index-set row              */
  int32_t block;  /* 0/1: token-level argsTopK; else positions per selected block */
} lychee_shape;

/* Bytes of device workspace that serve both lychee_hybrid_decode_attn and
 * lychee_decode_stack for shape *s (any L).  Returns 0 if *s is invalid.  The
 * workspace holds fp32 logits of retrieval heads ([B, Hq, N_max], the raw dot
 * products q.k, not divided by sqrt(d)), split partials, one membership bitmap
 * per head position ([B, Hq, ceil(N_max/32)] uint32, bit j of word w =
 * position 32w+j is in S), work counters and the device error word.  The
 * stack keeps two logits regions and three partial-state regions, so that a
 * layer's attention overlaps the previous layer's selection and combine. */
LYCHEE_API size_t lychee_workspace_size(const lychee_shape* s);

/* Bytes of device workspace that lychee_hybrid_decode_attn alone needs for
 * shape *s: the leading part of lychee_workspace_size(s) (one logits region,
 * one partial-state region, the bitmaps).  Returns 0 if *s is invalid. */
LYCHEE_API size_t lychee_layer_workspace_size(const lychee_shape* s);

/* Byte offsets, inside a workspace for shape *s, of the fp32 logits region
 * [B, Hq, N_max] (raw q.k of the retrieval heads of the most recent
 * lychee_hybrid_decode_attn call, positions j < n_b; the stack alternates
 * between this region and another) and of the membership-bitmap region [B, Hq, nwords]
 * (nwords = ceil(N_max / 32)); *nwords receives nwords.  For inspection and
 * tests.  Returns LYCHEE_ERR_INVALID_ARG for an invalid shape or NULL output. */
LYCHEE_API lychee_status lychee_workspace_offsets(const lychee_shape* s, size_t* logits_off,
                                                  size_t* bitmaps_off, int32_t* nwords);

/* One hybrid-head layer (method steps (3) and (4)).
 *   q         device [B, Hq, d]          dtype
 *   k_cache   device [B, Hkv, N_max, d]  dtype, rows j < n_b hold the cache
 *   v_cache   device [B, Hkv, N_max, d]  dtype
 *   seqlens   device [B] int32, 1 <= n_b <= N_max (the current token is included)
 *   k_per_seq device [B] int32 or NULL (then k_b = min(k, n_b))
 *   head_role HOST   [Hq] uint8, LYCHEE_ROLE_RETRIEVAL or LYCHEE_ROLE_SPARSE
 *   idx_in    device [B, Hq, k] int32; rows of sparse heads are read (their
 *             entries before the first -1, at most k_b of them, strictly
 *             ascending, in [0, n_b)); may be NULL only when every head is a
 *             retrieval head.  A block-granular set may hold more than k_b
 *             positions (k_b < block); this call reads only its first k_b,
 *             whereas lychee_decode_stack hands every set on whole
 *   out       device [B, Hq, d] dtype
 *   idx_out   device [B, Hq, k] int32: retrieval heads get argsTopK of their
 *             logits, or their block-granular set (s->block), ascending, -1
 *             padded; sparse heads get their idx_in row copied bit for bit
 *   workspace device, >= lychee_layer_workspace_size(s) bytes, 256-byte aligned
 *   stream    cudaStream_t
 * The call overwrites the whole workspace header, so device errors reported by
 * lychee_check_device_error() refer to the most recent call on that workspace. */
LYCHEE_API lychee_status lychee_hybrid_decode_attn(const lychee_shape* s, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* seqlens, const int32_t* k_per_seq,
                                        const uint8_t* head_role, const int32_t* idx_in,
                                        void* out, int32_t* idx_out, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Size of the static device scratch behind lychee_hybrid_decode_attn_noalloc:
 * 64 MiB per device, enough for a layer whose lychee_layer_workspace_size() is
 * at most that (e.g. B = 1, Hq = 32, d = 128, N_max = 131072 needs about 49 MiB). */
#define LYCHEE_NOALLOC_SCRATCH_BYTES (64u << 20)

/* lychee_hybrid_decode_attn without a caller-owned workspace and without any
 * device allocation.  The method has no counterpart to this call: it is a
 * convenience of the library boundary for callers that may not allocate.
 * Arguments q .. idx_out and stream are those of lychee_hybrid_decode_attn and
 * the results are the same, bit for bit.  The workspace is a file-scope
 * __device__ array of LYCHEE_NOALLOC_SCRATCH_BYTES (one per device, part of the
 * library's device code); the call allocates nothing, and clears the part of the
 * scratch that must start at zero (error word, work counters) itself.
 *   device_error device uint32 or NULL: receives, in stream order, the device
 *                error bits of this call (as lychee_check_device_error's detail)
 * Returns LYCHEE_ERR_WORKSPACE, before touching the GPU, when
 * lychee_layer_workspace_size(s) exceeds LYCHEE_NOALLOC_SCRATCH_BYTES; the shape and
 * argument errors of lychee_hybrid_decode_attn otherwise; LYCHEE_ERR_CUDA if the
 * scratch address cannot be looked up.
 * All calls in one CUDA context (one per device and process) share the
 * scratch: calls whose executions overlap (other streams, host threads) race on
 * it, so serialise them.  The first call on each device looks the scratch
 * address up (cudaGetSymbolAddress); make it before any stream capture.  The
 * address is remembered per device together with the context it was looked up
 * in, and looked up again when the device's current context has changed (after
 * cudaDeviceReset, say). */
LYCHEE_API lychee_status lychee_hybrid_decode_attn_noalloc(const lychee_shape* s, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* seqlens, const int32_t* k_per_seq,
                                        const uint8_t* head_role, const int32_t* idx_in,
                                        void* out, int32_t* idx_out, uint32_t* device_error,
                                        void* stream);

/* L chained layers of one decode step (method steps (1), (3), (4)): the set
 * leaving head position h of layer l is the incoming set of head position h of
 * layer l+1; it is carried between layers as the per-head bitmap in the
 * workspace.
 *   q          device [L, B, Hq, d] dtype (one query per layer)
 *   k_caches   HOST array of L device pointers, each [B, Hkv, N_max, d]
 *   v_caches   HOST array of L device pointers, each [B, Hkv, N_max, d]
 *   seqlens    device [B]; k_per_seq device [B] or NULL (as above)
 *   head_role  HOST [L, Hq] uint8; row 0 must be all retrieval
 *   out        device [L, B, Hq, d] dtype
 *   idx_final  device [B, Hq, k] int32: the sets leaving layer L-1
 *   idx_layers device [L, B, Hq, k] int32 or NULL: the sets leaving every layer
 *   workspace, stream as above. */
LYCHEE_API lychee_status lychee_decode_stack(const lychee_shape* s, int32_t L, const void* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seqlens, const int32_t* k_per_seq,
                                  const uint8_t* head_role, void* out, int32_t* idx_final,
                                  int32_t* idx_layers, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* lychee_hybrid_decode_attn with a sliding-window branch on every sparse head,
 * fused with its sparse branch by a sigmoid gate (page "HySparse: A Hybrid
 * Sparse Attention Architecture with Oracle Token Selection and KV Cache
 * Sharing", paperlayer.ai/abs/2602.03560v1, Methodology: sparse layers combine
 * the sparse branch with a local sliding-window branch -- window 128, its own
 * cache -- through sigmoid gating).  For a sparse head h of KV group g:
 *   O_window = softmax(q_h . K_w^T / sqrt(d)) V_w over the min(window, n_b)
 *              rows in use of the group's window ring,
 *   out_h    = s * O_sparse + (1 - s) * O_window,  s = 1 / (1 + exp(-gate[b, h])).
 * Retrieval heads are unchanged.  Extra arguments (the rest as in
 * lychee_hybrid_decode_attn, whose results this gives for retrieval heads and
 * for sets, bit for bit):
 *   swa_k, swa_v device [B, Hkv, window, d] dtype, 16-byte aligned: the window
 *                ring of each sequence and KV group, position j in row
 *                j % window (rows 0 .. min(window, n_b) - 1 are read)
 *   window       1 .. 1024 (the page's choice is 128)
 *   gate         device [B, Hq] fp32 gate logits (read for sparse heads)
 * Arithmetic: fp32 scores of exact products, fp32 softmax and sums. */
LYCHEE_API lychee_status lychee_hybrid_decode_attn_swa(const lychee_shape* s, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* seqlens, const int32_t* k_per_seq,
                                        const uint8_t* head_role, const int32_t* idx_in,
                                        const void* swa_k, const void* swa_v, int32_t window,
                                        const float* gate, void* out, int32_t* idx_out,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* lychee_decode_stack with the sliding-window branch of
 * lychee_hybrid_decode_attn_swa on the sparse heads of every layer.
 *   swa_k, swa_v HOST arrays of L device pointers, each [B, Hkv, window, d]
 *   window       1 .. 1024
 *   gate         device [L, B, Hq] fp32 gate logits
 * The sets handed between layers do not depend on the window branch. */
LYCHEE_API lychee_status lychee_decode_stack_swa(const lychee_shape* s, int32_t L, const void* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seqlens, const int32_t* k_per_seq,
                                  const uint8_t* head_role, const void* const* swa_k,
                                  const void* const* swa_v, int32_t window, const float* gate,
                                  void* out, int32_t* idx_final, int32_t* idx_layers,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* The step before a layer's attention in a decode step: the current token's
 * key and value rows go into the caches at row n_b - 1 of their sequence (the
 * calls above read rows j < n_b, the current token included).  The rows are
 * copied bit for bit; the method's pages describe decoding over a KV cache
 * that holds the current token but give no rule of their own for the append.
 *   k_new, v_new      device [B, Hkv, d]         dtype
 *   k_cache, v_cache  device [B, Hkv, N_max, d]  dtype
 *   seqlens           device [B] int32; a sequence whose n_b is outside
 *                     [1, N_max] is left untouched
 *   stream            cudaStream_t
 * Only s->B, Hkv, d, N_max, dtype are used (the rest must still form a valid
 * shape).  Allocates nothing; graph-capturable.  The attention output `out`
 * [B, Hq, d] of the calls above is, byte for byte, the row-major [B, Hq * d]
 * matrix an output projection reads: no re-layout step is needed. */
LYCHEE_API lychee_status lychee_append_kv(const lychee_shape* s, const void* k_new,
                                          const void* v_new, void* k_cache, void* v_cache,
                                          const int32_t* seqlens, void* stream);

/* Head roles from HardKuma gate parameters (method steps (1), (2), (7) and the
 * closed-form expected L0 norm of the same page's novelty paragraph).  The gate
 * of head h in layer l is z ~ HardKuma(alpha, beta): K ~ Kumaraswamy(alpha,
 * beta) on (0, 1) with CDF F(x) = 1 - (1 - x^alpha)^beta, stretched to
 * p + (q - p) K and rectified to [0, 1].  A head is a retrieval head when
 * E[z] > 0.5; with layer0_retrieval, layer 0 is all retrieval whatever its
 * parameters.  The expected L0 norm is the sum over the gated heads (every head
 * but layer 0's when layer0_retrieval) of P(z != 0) = 1 - F(-p / (q - p)).
 * Computed in fp64; E[z] by the integral (q - p) * integral_a^b (1 - k^alpha)^beta dk,
 * a = -p/(q-p), b = (1-p)/(q-p), with composite Simpson's rule (2048 panels).
 *   alpha, beta  device [L, Hq] double, finite and > 0 (a head with other values
 *                gets E[z] = NaN and the sparse role, and makes the L0 sum NaN)
 *   p, q         stretch limits, p < 0 and q > 1 (the HardKuma distribution's
 *                usual choice is p = -0.1, q = 1.1; the pages give none)
 *   head_role    device [L, Hq] uint8 out: LYCHEE_ROLE_RETRIEVAL / _SPARSE, the
 *                form lychee_decode_stack takes (after a copy to the host)
 *   expected_z   device [L, Hq] double out, or NULL
 *   expected_l0  device [1] double out, or NULL
 * Returns LYCHEE_ERR_INVALID_ARG for NULL inputs, L or Hq below 1, p >= 0,
 * q <= 1 or pointers not 8-byte aligned; allocates nothing; one launch. */
LYCHEE_API lychee_status lychee_hardkuma_roles(const double* alpha, const double* beta, int32_t L,
                                               int32_t Hq, double p, double q,
                                               int32_t layer0_retrieval, uint8_t* head_role,
                                               double* expected_z, double* expected_l0,
                                               void* stream);

/* Synchronises `stream`, reads the device error word of `workspace` and clears
 * it.  Returns LYCHEE_OK, LYCHEE_ERR_BAD_INDEX, LYCHEE_ERR_TIMEOUT or
 * LYCHEE_ERR_CUDA.  If detail is not NULL it receives the raw flag bits
 * (1 = bad index, 2 = bad sequence length, 4 = bad budget, 8 = wait timeout). */
LYCHEE_API lychee_status lychee_check_device_error(void* workspace, void* stream, uint32_t* detail);

/* Static, NUL-terminated description of a status code. */
LYCHEE_API const char* lychee_status_string(lychee_status st);

/* Library version as 10000*major + 100*minor + patch. */
LYCHEE_API int32_t lychee_version(void);

/* Launch profiler (measurement aid, off by default).  Between begin and end,
 * every kernel launch of the library on any stream is bracketed by two CUDA
 * events recorded on its launch stream, up to max_launches launches (later
 * launches run unrecorded).  lychee_profile_end synchronises on the recorded
 * events and writes, for the first min(n, capacity) launches, the kind
 * (0 attention, 1 top-k, 2 combine, 3 set->bitmap, 4 bitmap->set, 5 the
 * retrieval heads' selection -- argsTopK, or the block selection when
 * s->block > 1 -- and the combine in one launch; in a stack, 1 is the
 * selection alone) and the
 * elapsed milliseconds; *n_out receives n.  Process-global state: one profiling
 * session at a time.  Events are created on the current device on first use
 * and kept for reuse. */
LYCHEE_API lychee_status lychee_profile_begin(int32_t max_launches);
/* Span mode of the same profiler: no events between launches (the layers of a
 * stack still overlap), but per lychee_decode_stack(_swa) call two events, one
 * before its first attention launch and one after its last, up to max_spans
 * calls; lychee_profile_end reports each as kind 6 with the milliseconds
 * between them (the time the call's attention launches take, back to back,
 * with the selections that overlap them). */
LYCHEE_API lychee_status lychee_profile_spans_begin(int32_t max_spans);
LYCHEE_API lychee_status lychee_profile_end(int32_t capacity, int32_t* kinds, float* ms, int32_t* n_out);

#ifdef __cplusplus
}
#endif

#endif /* LYCHEE_H */
