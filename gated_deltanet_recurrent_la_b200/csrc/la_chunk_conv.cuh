// la_chunk_conv.cuh -- the short causal convolution of the chunked prefill as a launch of
// its own: every (chunk, state head) tile independently (the window of a chunk's first
// tokens is the previous raw rows of its sequence, read from global memory, or the history
// at the sequence's read slot), its convolved q, k, v written per state head to a
// workspace that the one-launch chunked kernel then reads as its q, k and v.
//
// Per tile: one CTA of 192 threads; the chunk's raw q, k, v rows land in a shared-memory tile
// [64 tokens][384 channels] (cp.async), then thread i convolves the channel pair
// (2 (i % 64), 2 (i % 64) + 1) of q (i < 64), k (i < 128) or v in place, y_t = sum_j w[j]
// x_{t-W+1+j}, SiLU when asked, rounded to BF16; then q_t and k_t to unit length
// from the rounded rows (when asked); the tile leaves as 16-byte pieces of whole rows.  The
// tile holding a sequence's last token also writes its history (the last W - 1 raw inputs,
// earlier history entries when the sequence is shorter), and empty sequences pass their
// history through.
#pragma once

#include <cstdint>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {
namespace cconv {
constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kCH = 3 * kD;                   // q, k, v channels of a state head
constexpr int kThreads = 192;                 // one channel pair each
constexpr int kRowB = kCH * 2 + 16;           // padded row of the BF16 tile (bytes)
constexpr int kOffTile = 0;                   // [64][kCH] bf16 (rows kRowB apart)
constexpr int kOffNorm = kOffTile + kC * kRowB;  // 1 / |q_t|, 1 / |k_t|  [2][64] fp32
constexpr int kSmem = kOffNorm + 2 * kC * 4;
constexpr int kWsHeadBytes = 256;
}  // namespace cconv

// workspace: a 256-byte header, then the convolved q, k and v, each [T][H_v][128] BF16
inline size_t chunk_conv_workspace_bytes_impl(int64_t total_tokens, int64_t n_v_heads) {
  if (total_tokens < 0 || n_v_heads <= 0) return 0;
  return (size_t)(cconv::kWsHeadBytes + 3 * total_tokens * n_v_heads * cconv::kD * 2);
}

__global__ void __launch_bounds__(cconv::kThreads) chunk_conv_kernel(const ScanParams p) {
  using namespace cconv;
  extern __shared__ __align__(1024) unsigned char smem[];
  float* rnorm = reinterpret_cast<float*>(smem + kOffNorm);
  const int tid = threadIdx.x;
  const int m = tid / 64, pr = tid % 64;  // q, k or v; channel pair
  const int H = p.n_v_heads;
  const int ratio = H / p.n_qk_heads;
  const int wid = p.conv_w;
  const __nv_bfloat16* xq = static_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* xk = static_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* xv = static_cast<const __nv_bfloat16*>(p.v);
  __nv_bfloat16* ws = static_cast<__nv_bfloat16*>(const_cast<void*>(p.workspace)) + kWsHeadBytes / 2;
  const int64_t plane = (int64_t)p.total_tokens * H * kD;  // elements of each of q, k, v
  const __nv_bfloat16* hist_src = static_cast<const __nv_bfloat16*>(p.conv_src);
  __nv_bfloat16* hist_dst = static_cast<__nv_bfloat16*>(p.conv_dst);

  // empty sequences pass their history through (zero without a read slot)
  for (int s = blockIdx.x; s < p.n_seqs; s += gridDim.x) {
    const int t0 = __ldg(p.cu_seqlens + s), t1 = __ldg(p.cu_seqlens + s + 1);
    if (t1 != t0) continue;
    const int rs = p.read_slot ? __ldg(p.read_slot + s) : 0;
    const int wsl = p.write_slot ? __ldg(p.write_slot + s) : s;
    if ((p.read_slot && (rs < 0 || rs >= p.src_slots)) || wsl < 0 || wsl >= p.dst_slots) continue;
    for (int idx = tid; idx < H * kCH * (wid - 1); idx += kThreads) {
      const int h = idx / (kCH * (wid - 1)), r = idx % (kCH * (wid - 1));
      hist_dst[((int64_t)wsl * H + h) * kCH * (wid - 1) + r] =
          p.read_slot ? hist_src[((int64_t)rs * H + h) * kCH * (wid - 1) + r] : __float2bfloat16_rn(0.0f);
    }
  }

  const int64_t n_tiles = (int64_t)(p.total_tokens + kC - 1) / kC + p.n_seqs + 1;
  const int64_t items = n_tiles * H;
#pragma unroll 1
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int gc = (int)(item / H), h = (int)(item % H), hq = h / ratio;
    // the sequence of tile gc: the last s with cu[s] / 64 + s <= gc
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.cu_seqlens + mid) / kC + mid <= gc) lo = mid; else hi = mid - 1;
    }
    const int seq = lo;
    const int t0 = __ldg(p.cu_seqlens + seq), t1 = __ldg(p.cu_seqlens + seq + 1);
    if (t0 < 0 || t1 < t0 || t1 > p.total_tokens) continue;  // reported by the chunked launch
    const int c0 = (gc - (t0 / kC + seq)) * kC;
    if (c0 < 0 || c0 >= t1 - t0) continue;                   // a tile index no chunk uses
    const int ns = min(kC, t1 - t0 - c0);
    const int rs = p.read_slot ? __ldg(p.read_slot + seq) : 0;
    const int wsl = p.write_slot ? __ldg(p.write_slot + seq) : seq;
    if ((p.read_slot && (rs < 0 || rs >= p.src_slots)) || wsl < 0 || wsl >= p.dst_slots) continue;

    // this thread's two channels: weights as four taps over the window of the last three raw
    // inputs and the current one, and that window at the chunk's start
    const int ch0 = m * kD + 2 * pr;  // channel within the head's q | k | v
    const __nv_bfloat16* xs = m == 0 ? xq + (int64_t)hq * kD : m == 1 ? xk + (int64_t)hq * kD : xv + (int64_t)h * kD;
    const int64_t xstride = (int64_t)(m == 2 ? H : p.n_qk_heads) * kD;
    const float* wsrc = (m == 0 ? p.conv_wq : m == 1 ? p.conv_wk : p.conv_wv) +
                        ((int64_t)(m == 2 ? h : hq) * kD + 2 * pr) * wid;
    float w[2][4], win[2][3];
    const __nv_bfloat16* hs = hist_src + ((int64_t)rs * H + h) * kCH * (wid - 1);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int tap = 0; tap < 4; ++tap) {
        const int src = tap - (4 - wid);  // tap multiplies x_{t-3+tap}
        w[e][tap] = src >= 0 ? __ldg(wsrc + e * wid + src) : 0.0f;
      }
#pragma unroll
      for (int sl = 0; sl < 3; ++sl) {
        // slot sl holds x_{c0-3+sl} of the sequence: a raw row, or history entry
        // (W - 1) + (c0 - 3 + sl) before the sequence's first token
        const int tt = c0 - 3 + sl;
        float v = 0.0f;
        if (tt >= 0) {
          v = __bfloat162float(xs[(int64_t)(t0 + tt) * xstride + 2 * pr + e]);
        } else {
          const int hidx = (wid - 1) + tt;
          if (hidx >= 0 && p.read_slot) v = __bfloat162float(hs[(ch0 + e) * (wid - 1) + hidx]);
        }
        win[e][sl] = v;
      }
    }
    // the chunk's raw rows into the tile (q | k | v of the head), then y in place, rounded to
    // BF16 (each thread reads and writes only its own channel pair)
    for (int idx = tid; idx < ns * 48; idx += kThreads) {
      const int tt = idx / 48, pc = idx % 48, mm = pc / 16;
      const __nv_bfloat16* src = (mm == 0 ? xq + (int64_t)hq * kD : mm == 1 ? xk + (int64_t)hq * kD : xv + (int64_t)h * kD) +
                                 (int64_t)(t0 + c0 + tt) * (mm == 2 ? H : p.n_qk_heads) * kD + (pc % 16) * 8;
      cp_async_16(smem + kOffTile + tt * kRowB + pc * 16, src);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < ns; ++t) {
      uint32_t* cell = reinterpret_cast<uint32_t*>(smem + kOffTile + t * kRowB + ch0 * 2);
      const uint32_t xr = *cell;
      float y[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float xin = e ? bf16_hi(xr) : bf16_lo(xr);
        float yy = fmaf(w[e][3], xin, fmaf(w[e][2], win[e][2], fmaf(w[e][1], win[e][1], w[e][0] * win[e][0])));
        win[e][0] = win[e][1];
        win[e][1] = win[e][2];
        win[e][2] = xin;
        if (p.conv_act) yy = __fdividef(yy, 1.0f + __expf(-yy));
        y[e] = yy;
      }
      *cell = pack_bf16x2(y[0], y[1]);
    }
    // the history after the sequence's last token (this tile holds it)
    if (c0 + ns == t1 - t0) {
      __nv_bfloat16* hd = hist_dst + ((int64_t)wsl * H + h) * kCH * (wid - 1);
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int sl = 0; sl < 3; ++sl) {
          const int dst = sl - (4 - wid);
          if (dst >= 0) hd[(ch0 + e) * (wid - 1) + dst] = __float2bfloat16_rn(win[e][sl]);
        }
    }
    __syncthreads();
    // q_t and k_t to unit length, from the rounded rows (thread: row t of q or k)
    if (p.conv_l2norm) {
      if (tid < 2 * kC) {
        const int t = tid % kC, qk = tid / kC;
        float ss = 0.0f;
        if (t < ns) {
#pragma unroll 4
          for (int pc = 0; pc < 16; ++pc) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(smem + kOffTile + t * kRowB + qk * kD * 2 + pc * 16);
            const uint32_t vw[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) ss = fmaf(bf16_lo(vw[e2]), bf16_lo(vw[e2]), fmaf(bf16_hi(vw[e2]), bf16_hi(vw[e2]), ss));
          }
        }
        rnorm[qk * kC + t] = rsqrtf(ss + 1e-6f);
      }
      __syncthreads();
    }
    // the tile to the workspace: q, k, v rows of head h as 16-byte pieces
    for (int idx = tid; idx < ns * 48; idx += kThreads) {
      const int t = idx / 48, pc = idx % 48, mm = pc / 16;
      uint4 v4 = *reinterpret_cast<const uint4*>(smem + kOffTile + t * kRowB + pc * 16);
      if (p.conv_l2norm && mm < 2) {
        const float r = rnorm[mm * kC + t];
        v4 = make_uint4(pack_bf16x2(bf16_lo(v4.x) * r, bf16_hi(v4.x) * r), pack_bf16x2(bf16_lo(v4.y) * r, bf16_hi(v4.y) * r),
                        pack_bf16x2(bf16_lo(v4.z) * r, bf16_hi(v4.z) * r), pack_bf16x2(bf16_lo(v4.w) * r, bf16_hi(v4.w) * r));
      }
      *reinterpret_cast<uint4*>(ws + mm * plane + ((int64_t)(t0 + c0 + t) * H + h) * kD + (pc % 16) * 8) = v4;
    }
    __syncthreads();  // the tile is read before the next item's writes
  }
}

}  // namespace la
