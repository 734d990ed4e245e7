// la_chunk_noalloc.cu -- the workspace of the two-launch chunked prefill as a fixed device
// array of the library itself, for callers that hand over no scratch buffer.  One array
// per device (the module is loaded on each device that uses it); its address comes from
// the runtime's symbol lookup on the current device, cached per device together with the
// identity of the context it was looked up in: after a device reset the next call runs in
// a new context and looks the address up again.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {

namespace {

constexpr size_t kNoAllocBytes = size_t(256) << 20;
static __device__ __align__(256) unsigned char g_chunk_workspace[kNoAllocBytes];

constexpr int kMaxDevices = 128;
std::mutex g_ws_mutex;
struct WsEntry {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;  // the context the address belongs to (0: none yet)
};
WsEntry g_ws[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Identity of the calling thread's current context (driver entry points looked up once
// through the runtime); 0 when it cannot be determined, which disables the cache.
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = []() -> CtxGetCurrentFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  static const CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetIdFn>(f);
  }();
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

cudaError_t chunk_noalloc_workspace(void** addr, size_t* bytes) {
  *addr = nullptr;
  *bytes = kNoAllocBytes;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  WsEntry& w = g_ws[dev];
  const unsigned long long ctx = current_context_id();
  if (w.addr == nullptr || ctx == 0 || ctx != w.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_chunk_workspace);
    if (e != cudaSuccess) {
      w.addr = nullptr;
      w.ctx_id = 0;
      return e;
    }
    w.addr = p;
    // the context is certainly current after the lookup; record it for the next call
    w.ctx_id = ctx != 0 ? ctx : current_context_id();
  }
  *addr = w.addr;
  return cudaSuccess;
}

}  // namespace la
