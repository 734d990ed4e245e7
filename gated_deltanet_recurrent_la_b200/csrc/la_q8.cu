// la_q8.cu -- conversion between FP32 states and the slots of a q8 pool (the mixed INT8 /
// BF16 storage of la_state.h, after the DAMP passage of "Seven Architectures Replacing KV
// Cache With Bounded Mutable State"): one CTA per (slot, head) tile, one warp per row at a
// time, lane j holding column 32 g + j of the row's group g, so a group's absmax is one
// warp reduction.  Codes are decided in FP32 with correctly rounded division and
// multiplication, the same arithmetic as the decode step and the scan.
#include <cstdint>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {

namespace {

constexpr int kCodecThreads = 256;

__global__ void __launch_bounds__(kCodecThreads) q8_codec_kernel(const Q8CodecParams p) {
  const int H = p.n_v_heads, DK = p.d_k, DV = p.d_v, NG = DV / 32, NW = DK / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n8 = DK - p.n_hp;
  const int64_t tile_bytes = q8_tile_bytes(DK, DV, p.n_hp);
  for (int64_t t = blockIdx.x; t < (int64_t)p.n * H; t += gridDim.x) {
    const int i = (int)(t / H), h = (int)(t % H);
    const int slot = __ldg(p.slots + i);
    if (slot < 0 || slot >= p.n_slots) {
      if (threadIdx.x == 0) report(p.err, p.encode ? LA_DEVERR_WRITE_SLOT : LA_DEVERR_READ_SLOT);
      continue;
    }
    uint32_t mk[4] = {0u, 0u, 0u, 0u};  // d_k <= 128
    int count = 0;
    for (int w = 0; w < NW; ++w) {
      mk[w] = __ldg(p.mask + h * NW + w);
      count += __popc(mk[w]);
    }
    if (count != p.n_hp) {
      if (threadIdx.x == 0) report(p.err, LA_DEVERR_Q8_MASK);
      continue;
    }
    unsigned char* tile = static_cast<unsigned char*>(p.pool) + ((int64_t)slot * H + h) * tile_bytes;
    float* x = p.dense + t * DK * DV;
    for (int row = warp; row < DK; row += kCodecThreads / 32) {
      // rank of the row among the BF16 rows and among the INT8 rows
      int below = 0;
      for (int w = 0; w < row / 32; ++w) below += __popc(mk[w]);
      below += __popc(mk[row / 32] & ((1u << (row % 32)) - 1u));
      const bool hp = (mk[row / 32] >> (row % 32)) & 1u;
      const int idx = hp ? below : row - below;
      __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(tile + n8 * DV + n8 * NG * 4) + (int64_t)idx * DV;
      int8_t* crow = reinterpret_cast<int8_t*>(tile) + (int64_t)idx * DV;
      float* srow = reinterpret_cast<float*>(tile + n8 * DV) + (int64_t)idx * NG;
      for (int g = 0; g < NG; ++g) {
        const int col = 32 * g + lane;
        if (p.encode) {
          const float v = x[(int64_t)row * DV + col];
          float amax = fabsf(v);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
          if (hp) {
            hrow[col] = __float2bfloat16_rn(v);
          } else {
            float s, inv;
            q8_scales(amax, s, inv);
            crow[col] = (int8_t)(int)q8_code(v, inv);
            if (lane == 0) srow[g] = s;
          }
        } else {
          x[(int64_t)row * DV + col] =
              hp ? __bfloat162float(hrow[col]) : __fmul_rn((float)crow[col], srow[g]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_q8_codec(const Q8CodecParams& p, cudaStream_t stream) {
  const int64_t tiles = (int64_t)p.n * p.n_v_heads;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  const int grid = (int)(tiles < cap ? tiles : (cap > 0 ? cap : 1));
  q8_codec_kernel<<<grid, kCodecThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace la
