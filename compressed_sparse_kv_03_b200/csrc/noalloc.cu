// Decode attention without caller-provided scratch.
//
// Callers that cannot allocate device memory -- for example a plugin running
// inside a serving engine that owns every allocation and only hands its
// plugins a stream, or real-time code that must not call cudaMalloc because it
// can synchronise the device and stall other streams -- still need the split-KV
// partials that csa_sparse_attn_decode keeps in its workspace.  This entry
// point gives them that scratch from a fixed array in the library's own device
// memory: it allocates nothing, and every GPU that loads the library holds the
// array until the process exits.
#include <cstdio>
#include <mutex>

#include "kernels.h"

namespace csa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

// The shared scratch.  In host code this name is only a handle: its device
// address comes from cudaGetSymbolAddress on each device.
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and kept for the life of the process.  A
// device reset (cudaDeviceReset, or anything else that destroys the primary
// context) unloads the module; the array may then sit at another address, so
// this form must not be called again in that process after such a reset.
csa_status_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_error("csa_sparse_attn_decode_noalloc: cudaGetDevice failed");
    return CSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_last_error("csa_sparse_attn_decode_noalloc: device ordinal beyond 63");
    return CSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char buf[160];
      snprintf(buf, sizeof(buf), "csa_sparse_attn_decode_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      set_last_error(buf);
      return CSA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA_OK;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" csa_status_t csa_sparse_attn_decode_noalloc(
    const csa_bf16* q, const csa_cache_t* kv_comp, const csa_bf16* win, const int32_t* win_len,
    const int32_t* idx, const int32_t* count, int32_t B, int32_t H, int32_t d, int32_t top_k,
    int32_t window, float sm_scale, const float* sink, csa_bf16* out, float* lse,
    csa_stream_t stream) {
  const char* name = "csa_sparse_attn_decode_noalloc";
  // every argument check comes before the scratch is looked up or touched, so
  // a rejected call enqueues nothing
  if (B == 0) return CSA_OK;
  csa_status_t st =
      check_decode_call(name, q, kv_comp, win, win_len, idx, count, B, H, d, top_k, window, out);
  if (st != CSA_OK) return st;
  const size_t need = csa_sparse_attn_decode_workspace_size(B, H, d, top_k, window);
  if (need > kNoAllocScratchBytes) {
    char buf[200];
    snprintf(buf, sizeof(buf),
             "csa_sparse_attn_decode_noalloc: this call needs %zu bytes of scratch, more than the "
             "%zu bytes of static scratch; use csa_sparse_attn_decode with a workspace",
             need, kNoAllocScratchBytes);
    set_last_error(buf);
    return CSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != CSA_OK) return st;
  // the device-check record at the head of the scratch must start clean
  cudaError_t e = cudaMemsetAsync(scratch, 0, kWsHeader, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_last_error("csa_sparse_attn_decode_noalloc: clearing the scratch header failed");
    return CSA_ERR_CUDA;
  }
  return csa_sparse_attn_decode(q, kv_comp, win, win_len, idx, count, B, H, d, top_k, window,
                                sm_scale, sink, out, lse, scratch, kNoAllocScratchBytes, stream,
                                nullptr);
}
