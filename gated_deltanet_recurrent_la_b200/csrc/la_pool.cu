// la_pool.cu -- whole-slot copies of the state pool (copy / gather / scatter / zero).
//
// Prefix-cache checkpoints ("Recurrent state" glossary page, Why it matters: separate
// read and write slots so a cached checkpoint survives) and snapshots for rollback or
// migration ("Seven Architectures ...", ONNX section) are bit copies of whole slots.
// One kernel serves all four: 16-byte vectors, four in flight per thread, each CTA
// moving one 16 KiB chunk of one slot per iteration of a grid-stride loop over
// (slot, chunk).  The result is bit-exact by construction (no arithmetic).
#include <algorithm>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {

namespace {

constexpr int kPoolThreads = 256;
constexpr int kPoolUnroll = 4;
constexpr int64_t kChunkVecs = (int64_t)kPoolThreads * kPoolUnroll;  // 16 KiB

__global__ void __launch_bounds__(kPoolThreads) pool_copy_kernel(const PoolCopyParams p) {
  const int64_t vecs = p.slot_bytes / 16;
  const int64_t chunks = (vecs + kChunkVecs - 1) / kChunkVecs;
  const int64_t work = (int64_t)p.n * chunks;
  for (int64_t w = blockIdx.x; w < work; w += gridDim.x) {
    const int i = (int)(w / chunks);
    const int64_t chunk = w % chunks;
    const int s = p.src_index ? __ldg(p.src_index + i) : i;
    const int d = p.dst_index ? __ldg(p.dst_index + i) : i;
    const bool s_ok = p.zero || (s >= 0 && s < p.src_count);
    const bool d_ok = d >= 0 && d < p.dst_count;
    if (!s_ok || !d_ok) {
      if (chunk == 0 && threadIdx.x == 0)
        report(p.err, (s_ok ? 0u : LA_DEVERR_READ_SLOT) | (d_ok ? 0u : LA_DEVERR_WRITE_SLOT));
      continue;
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<unsigned char*>(p.dst) + (int64_t)d * p.slot_bytes);
    const int64_t v0 = chunk * kChunkVecs + threadIdx.x;
    if (p.zero) {
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        const int64_t vi = v0 + (int64_t)u * kPoolThreads;
        if (vi < vecs) dst[vi] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      const uint4* src =
          reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.src) + (int64_t)s * p.slot_bytes);
      uint4 x[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        const int64_t vi = v0 + (int64_t)u * kPoolThreads;
        if (vi < vecs) x[u] = __ldcs(src + vi);
      }
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        const int64_t vi = v0 + (int64_t)u * kPoolThreads;
        if (vi < vecs) dst[vi] = x[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_pool_copy(const PoolCopyParams& p, cudaStream_t stream) {
  const int per_sm = prepare_kernel(reinterpret_cast<const void*>(&pool_copy_kernel), kPoolThreads, 0);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  const int64_t chunks = (p.slot_bytes / 16 + kChunkVecs - 1) / kChunkVecs;
  const int64_t work = (int64_t)p.n * chunks;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)std::min<int64_t>(work, cap);
  pool_copy_kernel<<<grid, kPoolThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace la
