// noalloc.cu -- lychee_hybrid_decode_attn served from a static device scratch,
// for callers that may not allocate device memory (or own no workspace).
//
// The scratch is one file-scope __device__ array, created with this file's
// module; its address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and cached.  Nothing here calls cudaMalloc,
// cudaFree or any routine that allocates.  Every call goes through
// lychee_hybrid_decode_attn unchanged, which first clears the workspace header
// (device error word and work counters, the only state that must start at
// zero); all other scratch regions are written before they are read.
//
// One scratch per device: two calls whose executions overlap (on different
// streams, host threads or processes' contexts sharing it) race on it.  The
// first call on a device does the address lookup, which must not run inside a
// stream capture, so make it before capturing any stream.
#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "lychee.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[LYCHEE_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use).
lychee_status current_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return LYCHEE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return LYCHEE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LYCHEE_OK;
}

}  // namespace

extern "C" LYCHEE_API lychee_status lychee_hybrid_decode_attn_noalloc(
    const lychee_shape* s, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* seqlens, const int32_t* k_per_seq, const uint8_t* head_role,
    const int32_t* idx_in, void* out, int32_t* idx_out, uint32_t* device_error, void* stream) {
  const size_t need = lychee_workspace_size(s);
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
