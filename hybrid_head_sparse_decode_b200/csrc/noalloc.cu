// noalloc.cu -- lychee_hybrid_decode_attn served from a static device scratch,
// for callers that may not allocate device memory (or own no workspace).
//
// The scratch is one file-scope __device__ array, created with this file's
// module in every CUDA context that loads the library; its address is looked
// up with cudaGetSymbolAddress (with the device current) and remembered per
// device together with the context it belongs to, and looked up again when the
// device's current context is another one (after cudaDeviceReset, say).
// Nothing here calls cudaMalloc, cudaFree or any routine that allocates.  Every
// call goes through lychee_hybrid_decode_attn unchanged, which first clears the
// workspace header (device error word and work counters, the only state that
// must start at zero); all other scratch regions are written before they are
// read.
//
// One scratch per context: two calls in one process whose executions overlap
// on a device (on different streams or host threads) race on it.  The first
// call on a device does the address lookup, which must not run inside a stream
// capture, so make it before capturing any stream.
#include <cudaTypedefs.h>

#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "lychee.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[LYCHEE_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent through the runtime's entry-point query (the
// library does not link libcuda); null if unavailable.
PFN_cuCtxGetCurrent_v4000 ctx_getter() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    cudaGetLastError();
  });
  return fn;
}

// Device address of g_scratch in the current device's current context.
lychee_status current_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return LYCHEE_ERR_CUDA;
  }
  PFN_cuCtxGetCurrent_v4000 get = ctx_getter();
  if (!get) return LYCHEE_ERR_CUDA;
  CUcontext ctx = nullptr;   // null until the runtime has made a context current
  if (get(&ctx) != CUDA_SUCCESS) return LYCHEE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);   // makes the context current
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return LYCHEE_ERR_CUDA;
    }
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return LYCHEE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return LYCHEE_OK;
}

}  // namespace

extern "C" LYCHEE_API lychee_status lychee_hybrid_decode_attn_noalloc(
    const lychee_shape* s, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* seqlens, const int32_t* k_per_seq, const uint8_t* head_role,
    const int32_t* idx_in, void* out, int32_t* idx_out, uint32_t* device_error, void* stream) {
  const size_t need = lychee_layer_workspace_size(s);
  if (need == 0)   // invalid shape: the layer call reports which check failed
    return lychee_hybrid_decode_attn(s, q, k_cache, v_cache, seqlens, k_per_seq, head_role,
                                     idx_in, out, idx_out, nullptr, 0, stream);
  if (need > (size_t)LYCHEE_NOALLOC_SCRATCH_BYTES) return LYCHEE_ERR_WORKSPACE;
  void* ws = nullptr;
  lychee_status st = current_scratch(&ws);
  if (st != LYCHEE_OK) return st;
  st = lychee_hybrid_decode_attn(s, q, k_cache, v_cache, seqlens, k_per_seq, head_role, idx_in,
                                 out, idx_out, ws, (size_t)LYCHEE_NOALLOC_SCRATCH_BYTES, stream);
  if (st != LYCHEE_OK || !device_error) return st;
  const char* err_word = static_cast<const char*>(ws) + offsetof(lychee::WsHeader, err);
  if (cudaMemcpyAsync(device_error, err_word, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LYCHEE_ERR_CUDA;
  }
  return LYCHEE_OK;
}
