// fix_attn_fwd_noalloc: the forward for callers that cannot allocate device
// memory.
//
// Some callers of this library have no way to obtain a device workspace at
// call time: host code that was handed only a stream and the tensors, or a
// runtime whose device memory is reserved up front and must not grow (an
// allocation there would fail, or synchronise the device).  For them this
// entry point runs the ordinary forward with its workspace placed in one
// file-scope device array of FIX_NOALLOC_MAX_WORKSPACE_BYTES, which every GPU
// that loads the library holds until the process exits.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress and caches it per device;
// make that first call before any stream capture.  Nothing here calls
// cudaMalloc, cudaFree or any allocating routine.
//
// Sharing: every call on a device uses the same array and leaves its contents
// behind.  The forward clears the one word that must start at zero (the
// device status word) and writes every other workspace byte before reading
// it.  Calls whose executions overlap on the GPU (different streams, or
// different host threads without ordering) race on the array.
//
// Status: the array's first word is the forward's device status word (where a
// bounded device wait that expired reports); fix_attn_noalloc_device_status
// reads it, since a caller of this entry point never sees the array's address.
#include <mutex>

#include "fix_attn.h"
#include <cuda_runtime.h>

static __device__ __align__(256) unsigned char fix_noalloc_scratch[FIX_NOALLOC_MAX_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch[kMaxDevices];  // device address of fix_noalloc_scratch, per device

// Device address of the scratch array on the current device (looked up once).
fix_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FIX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FIX_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, fix_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return FIX_ERR_CUDA;
    g_scratch[dev] = ptr;
  }
  *out = g_scratch[dev];
  return FIX_OK;
}

}  // namespace

extern "C" fix_status fix_attn_fwd_noalloc(const fix_attn_problem* p, const void* q,
                                           const void* k, const void* v, const float* g,
                                           const void* o_norm_weight, const void* o_gate,
                                           void* y, float* o_saved, float* m_saved,
                                           float* rstd_saved, void* stream) {
  const size_t need = fix_attn_workspace_bytes(p, 0);
  if (need == 0)  // invalid problem: let the forward report the exact reason
    return fix_attn_fwd(p, q, k, v, g, o_norm_weight, o_gate, y, o_saved, m_saved, rstd_saved,
                        nullptr, 0, stream);
  if (need > FIX_NOALLOC_MAX_WORKSPACE_BYTES) return FIX_ERR_WORKSPACE;
  void* ws = nullptr;
  const fix_status s = scratch_on_current_device(&ws);
  if (s != FIX_OK) return s;
  return fix_attn_fwd(p, q, k, v, g, o_norm_weight, o_gate, y, o_saved, m_saved, rstd_saved, ws,
                      FIX_NOALLOC_MAX_WORKSPACE_BYTES, stream);
}

extern "C" fix_status fix_attn_noalloc_device_status(void* stream) {
  void* ws = nullptr;
  const fix_status s = scratch_on_current_device(&ws);
  if (s != FIX_OK) return s;
  return fix_attn_device_status(ws, stream);
}
