// Decode attention without any caller-provided or allocated scratch.
//
// Some callers cannot hand this library a workspace: code running inside a
// host framework that owns every device allocation (a plugin may not call
// cudaMalloc), or code on a path where allocating would synchronise the
// device or is forbidden outright.  lrkv_decode_attn_static serves them: its
// scratch is a fixed array compiled into the library, held by every GPU that
// loads the library until the process exits.
//
// Host code must not use the array's name as a device pointer (on the host
// it names a host-side stand-in).  The first call on a device, with that
// device current, looks up the array's device address once with
// cudaGetSymbolAddress and keeps it; that first call should therefore come
// before any stream capture.  Every later call on the device reuses it, so
// the stream passed must belong to the current device, and a device reset
// (cudaDeviceReset) while the library is loaded is not supported: the kept
// address would be stale.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[LRKV_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LRKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LRKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return LRKV_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LRKV_OK;
}

}  // namespace

extern "C" int lrkv_decode_attn_static(const lrkv_cache* cache, const void* q,
                                       int32_t num_q_heads, const float* P_k, const float* P_v,
                                       int64_t basis_batch_stride, float scale, void* o,
                                       void* stream) {
  const size_t need = lrkv_decode_workspace_bytes(cache, num_q_heads);
  if (need == 0) {
    // the cache, the head counts or the plan were rejected: report why
    const int rc = lrkv::decode_plan_status(cache, num_q_heads);
    return rc != LRKV_OK ? rc : LRKV_ERR_ARG;
  }
  if (need > (size_t)LRKV_STATIC_WORKSPACE_BYTES) return LRKV_ERR_WORKSPACE;
  void* ws = nullptr;
  int rc = scratch_address(&ws);
  if (rc != LRKV_OK) return rc;
  // The array keeps the previous call's contents; only the error word in its
  // first bytes must start at zero, so clear it on the call's stream.
  if (cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LRKV_ERR_CUDA;
  return lrkv_decode_attn(cache, q, num_q_heads, P_k, P_v, basis_batch_stride, scale, o, ws,
                          (size_t)LRKV_STATIC_WORKSPACE_BYTES, stream);
}
