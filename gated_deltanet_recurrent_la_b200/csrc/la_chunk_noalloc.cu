// la_chunk_noalloc.cu -- the workspace of the two-launch chunked prefill as a fixed device
// array of the library itself, for callers that hand over no scratch buffer.  One array
// per device (the module is loaded on each device that uses it); its address comes from
// the runtime's symbol lookup on the current device.
#include <mutex>

#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {

namespace {

constexpr size_t kNoAllocBytes = size_t(256) << 20;
static __device__ __align__(256) unsigned char g_chunk_workspace[kNoAllocBytes];

constexpr int kMaxDevices = 128;
std::mutex g_ws_mutex;
void* g_ws_addr[kMaxDevices] = {nullptr};

}  // namespace

void* chunk_noalloc_workspace(size_t* bytes) {
  *bytes = kNoAllocBytes;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (!g_ws_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_chunk_workspace) != cudaSuccess) return nullptr;
    g_ws_addr[dev] = p;
  }
  return g_ws_addr[dev];
}

}  // namespace la
