// la_chunk.cuh -- chunked (WY / UT-transform) prefill on tensor cores.
//
// The same recurrence as la_scan.cuh, evaluated 64 tokens at a time so that its bulk
// becomes dense products ("Seven Architectures Replacing KV Cache With Bounded Mutable
// State": the "Kimi Linear" section's chunkwise-parallel kernel, the "Gated DeltaNet-2"
// section's chunkwise WY algorithm).  Per (sequence, head) and chunk of C tokens, with
// S0 the state at the chunk start, gamma_t the product of the chunk's gates up to token
// t, and (for the delta rules) beta:
//
//   L  = strictly-lower( beta_t (gamma_t / gamma_s) k_t . k_s )          C x C
//   T  = (I + L)^-1                                                      C x C
//   W  = T diag(beta gamma) K,   U~ = T diag(beta) V                     C x d_k, C x d_v
//   U  = U~ - W S0                                   (the per-token write vectors u_t)
//   O  = scale ( diag(gamma) Q S0 + (Q K^T (.) M) U ),  M_ts = gamma_t / gamma_s, s <= t
//   S  = gamma_C S0 + K^T diag(gamma_C / gamma) U
//
// which unrolls u_t = b (v_t - c S_{t-1}^T k_t), S_t = a S_{t-1} + k_t u_t^T exactly (the
// linear and gated rules have U = V).  Gate ratios use log|g| and a sign product, so
// negative gates are allowed.  Products take BF16 operands with FP32 accumulation; the
// FP32 state stays on chip (in tensor memory) across the whole sequence.
//
// This file: the definitions shared by the chunked kernels (d_k = d_v = 128, BF16
// q/k/v/o) and the intra-chunk launch of the two-launch form (chunk_prep_kernel).  The
// one-launch form is la_chunk_fused.cuh, the recurrence of the two-launch form
// la_chunk_tc.cuh.
#pragma once

#include <cstdint>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {
namespace chunk {

constexpr int kC = 64;         // tokens per chunk
constexpr int kD = 128;        // d_k = d_v

// shared-memory layout (bytes)
constexpr int kRow128 = kD * 2;                 // one BF16 row of 128
constexpr int kRow64 = kC * 2;                  // one BF16 row of 64
constexpr int kLs = kC + 4;                     // padded row stride of the FP32 L matrix
// workspace tile of one (chunk, head): Tw then Tu, [64][64] BF16 each, rows 128 bytes
// apart with the 16-byte piece c of row r at c ^ (r & 7); then the gate block, FP32
// [6][64] = gamma_t, gamma_C / gamma_t, A_t = gamma_t / e^m, B_t = e^m / gamma_t,
// log |gamma_t|, sign gamma_t, and one word that is 1 when gamma_t / gamma_s = A_t B_s
// may be used (the chunk's gates are at most 1 in magnitude and span at most e^80)
constexpr int kGateBlockBytes = (6 * kC + 4) * 4;
constexpr int kPrepTileBytes = 2 * kC * kRow64 + kGateBlockBytes;
// the workspace starts with a 256-byte header: word 0 counts the (sequence, head) units the
// recurrence launch has handed out (the prep launch zeroes it); the tiles follow
constexpr int kWsHeadBytes = 256;

// byte offset of the 16-byte chunk `ch` of row `r` in a swizzled matrix with rows of `rowb` bytes
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int ch, int rowb) {
  return base + r * rowb + ((ch ^ (r & 7)) << 4);
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A (16x16 bf16, row) * B (16x8 bf16, col), FP32 accumulate
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A (16x8 tf32, row) * B (8x8 tf32, col), FP32 accumulate; operands are FP32 bit patterns
__device__ __forceinline__ void mma1688_tf32(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc[2][4] (a 16 x 16 block as two 16 x 8 tiles) += A (16 x 16 at a, row stride lda) *
// B (16 x 16 at b, row stride ldb), FP32 row-major operands in shared memory, TF32 MMA
__device__ __forceinline__ void mma16x16x16_tf32(float (*acc)[4], const float* a, int lda, const float* b, int ldb,
                                                 int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 16; ks += 8) {
    uint32_t af[4];
    af[0] = __float_as_uint(a[g * lda + ks + t]);
    af[1] = __float_as_uint(a[(g + 8) * lda + ks + t]);
    af[2] = __float_as_uint(a[g * lda + ks + t + 4]);
    af[3] = __float_as_uint(a[(g + 8) * lda + ks + t + 4]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint32_t b0 = __float_as_uint(b[(ks + t) * ldb + 8 * nt + g]);
      const uint32_t b1 = __float_as_uint(b[(ks + t + 4) * ldb + 8 * nt + g]);
      mma1688_tf32(acc[nt], af, b0, b1);
    }
  }
}

// A fragment (rows m0..m0+15, k0..k0+15) of a row-major [m][k] matrix
__device__ __forceinline__ void lda(uint32_t* a, uint32_t base, int rowb, int m0, int k0, int lane) {
  ldsm4(swz(base, m0 + (lane & 15), (k0 >> 3) + (lane >> 4), rowb), a[0], a[1], a[2], a[3]);
}
// B fragments of two n-tiles (n0..n0+15, k0..k0+15) where B[k][n] = X[n][k], X row-major [n][k]
__device__ __forceinline__ void ldb_nk(uint32_t* b, uint32_t base, int rowb, int n0, int k0, int lane) {
  ldsm4(swz(base, n0 + (lane & 7) + ((lane >> 4) << 3), (k0 >> 3) + ((lane >> 3) & 1), rowb), b[0], b[1], b[2],
        b[3]);
}

// T = (I + L)^-1 in place of the strictly lower L ([64][kLs] FP32, rows kLs floats apart;
// the upper triangle of each diagonal 16 x 16 block zero, the blocks above the diagonal
// never read), by the 4 warps of a group (wi = 0..3, lane) that meet on the named barrier
// nb of 128 threads; sX is [3][16][kXs] FP32 scratch.  Diagonal block wi by forward
// substitution, lane c (and c + 16) owning column c (the column starts at zero, so full
// 16-term rows are exact); then block row bi of T from T_{bi,bj} = -D_bi sum_{bk=bj}^{bi-1}
// L_{bi,bk} T_{bk,bj}, warp bj < bi, on TF32 MMAs.
constexpr int kXs = 24;
__device__ __forceinline__ void ut_inverse64(float* sL, float* sX, int wi, int lane, uint32_t nb) {
  {
    const int b0 = 16 * wi, cc = lane & 15;
    float xc[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) xc[q] = 0.0f;
    const float4* lr = reinterpret_cast<const float4*>(sL + b0 * kLs + b0);
    float4 l0 = lr[0], l1 = lr[1], l2 = lr[2], l3 = lr[3];
#pragma unroll 1
    for (int rr = 0; rr < 16; ++rr) {
      // the next row's L while this row's sums run
      const float4* ln = reinterpret_cast<const float4*>(sL + (b0 + (rr < 15 ? rr + 1 : rr)) * kLs + b0);
      const float4 n0 = ln[0], n1 = ln[1], n2 = ln[2], n3 = ln[3];
      const float a0 = fmaf(l0.x, xc[0], fmaf(l0.y, xc[1], fmaf(l0.z, xc[2], l0.w * xc[3])));
      const float a1 = fmaf(l1.x, xc[4], fmaf(l1.y, xc[5], fmaf(l1.z, xc[6], l1.w * xc[7])));
      const float a2 = fmaf(l2.x, xc[8], fmaf(l2.y, xc[9], fmaf(l2.z, xc[10], l2.w * xc[11])));
      const float a3 = fmaf(l3.x, xc[12], fmaf(l3.y, xc[13], fmaf(l3.z, xc[14], l3.w * xc[15])));
      const float xv = (rr == cc ? 1.0f : 0.0f) - ((a0 + a1) + (a2 + a3));
#pragma unroll
      for (int q = 0; q < 16; ++q) xc[q] = (q == rr) ? xv : xc[q];
      l0 = n0;
      l1 = n1;
      l2 = n2;
      l3 = n3;
    }
    __syncwarp();
    if (lane < 16) {
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) sL[(b0 + rr) * kLs + b0 + cc] = xc[rr];
    }
  }
  named_bar_sync(nb, 128);
  // block row bi: T_{bi,bj} = -D_bi sum_{bk=bj}^{bi-1} L_{bi,bk} T_{bk,bj}, warp bj < bi
#pragma unroll 1
  for (int bi = 1; bi < 4; ++bi) {
    float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (wi < bi) {
      const int bj = wi;
      const int g8 = lane >> 2, t4 = lane & 3;
      float xs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 1
      for (int bk = bj; bk < bi; ++bk)
        mma16x16x16_tf32(xs, sL + (16 * bi) * kLs + 16 * bk, kLs, sL + (16 * bk) * kLs + 16 * bj,
                                kLs, lane);
      float* xw = sX + wi * 16 * kXs;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(xw + g8 * kXs + 8 * nt + 2 * t4) = make_float2(xs[nt][0], xs[nt][1]);
        *reinterpret_cast<float2*>(xw + (g8 + 8) * kXs + 8 * nt + 2 * t4) = make_float2(xs[nt][2], xs[nt][3]);
      }
      __syncwarp();
      mma16x16x16_tf32(y, sL + (16 * bi) * kLs + 16 * bi, kLs, xw, kXs, lane);
    }
    named_bar_sync(nb, 128);  // row bi of L is read: its blocks may now take T
    if (wi < bi) {
      const int bj = wi;
      const int g8 = lane >> 2, t4 = lane & 3;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int col = 16 * bj + 8 * nt + 2 * t4;
        *reinterpret_cast<float2*>(sL + (16 * bi + g8) * kLs + col) = make_float2(-y[nt][0], -y[nt][1]);
        *reinterpret_cast<float2*>(sL + (16 * bi + g8 + 8) * kLs + col) = make_float2(-y[nt][2], -y[nt][3]);
      }
    }
    named_bar_sync(nb, 128);
  }
}
}  // namespace chunk

// ---- the intra-chunk part on its own, per (chunk, head) tile: K K^T, the UT inverse
//      T = (I + L)^-1 by forward substitution in FP32 (one column of T per lane),
//      Tw = T diag(b gamma), Tu = T diag(b) and the chunk's gate block, written to the
//      workspace for chunk_tc_kernel.  Tiles are independent: a CTA of two warps takes one
//      at a time and several CTAs share an SM.  Chunk c of sequence s is workspace tile
//      (t0_s + 64 c) / 64 + s (distinct for every chunk; fewer than T / 64 + n_seqs + 1).
namespace chunk {
constexpr int kPThreads = 64;
constexpr int kPOffK = 0;                          // K [64][128] bf16, swizzled; then Tw, Tu [64][64]
constexpr int kPOffGB = kPOffK + kC * kRow128;     // the gate block (Tw, Tu, gate block = the tile)
constexpr int kPOffL = kPOffGB + kGateBlockBytes;  // L [64][68] fp32
constexpr int kPOffB = kPOffL + kC * kLs * 4;      // b_t [64]
constexpr int kPOffGin = kPOffB + kC * 4;          // g, beta [2][64]
constexpr int kPSmem = kPOffGin + 2 * kC * 4;
static_assert(2 * kC * kRow64 == kC * kRow128 && kPOffGB == 2 * kC * kRow64, "Tw, Tu take the K space");
static_assert(kPOffL % 16 == 0, "L rows are read as float4");
}  // namespace chunk

template <int RULE>
__global__ void __launch_bounds__(chunk::kPThreads) chunk_prep_kernel(const ScanParams p) {
  using namespace chunk;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_addr(smem);
  float* sL = reinterpret_cast<float*>(smem + kPOffL);
  float* gbk = reinterpret_cast<float*>(smem + kPOffGB);
  float* sBt = reinterpret_cast<float*>(smem + kPOffB);
  float* gin = reinterpret_cast<float*>(smem + kPOffGin);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int H = p.n_v_heads;
  const int ratio_h = H / p.n_qk_heads;
  if (blockIdx.x == 0 && tid == 0) *static_cast<unsigned int*>(const_cast<void*>(p.workspace)) = 0u;
  if (p.n_seqs <= 0) return;
  const int64_t n_tiles = (int64_t)(p.total_tokens + kC - 1) / kC + p.n_seqs + 1;
  const int64_t items = n_tiles * H;
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(p.k);

#pragma unroll 1
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int gc = (int)(item / H), h = (int)(item % H), hq = h / ratio_h;
    // the sequence of tile gc: the last s with cu[s] / 64 + s <= gc
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.cu_seqlens + mid) / kC + mid <= gc) lo = mid; else hi = mid - 1;
    }
    const int seq = lo;
    const int t0 = __ldg(p.cu_seqlens + seq), t1 = __ldg(p.cu_seqlens + seq + 1);
    if (t0 < 0 || t1 < t0 || t1 > p.total_tokens) continue;  // reported by the recurrence launch
    const int c0 = (gc - (t0 / kC + seq)) * kC;
    if (c0 < 0 || c0 >= t1 - t0) continue;                   // a tile index no chunk uses
    const int ns = (t1 - t0 - c0) < kC ? (t1 - t0 - c0) : kC;

    // K rows (zero beyond the sequence) and the gates ((1, 0) beyond it)
    for (int idx = tid; idx < kC * 16; idx += kPThreads) {
      const int r = idx >> 4, ch = idx & 15;
      unsigned char* d = smem + kPOffK + r * kRow128 + ((ch ^ (r & 7)) << 4);
      if (r < ns) cp_async_16(d, kg + ((int64_t)(t0 + c0 + r) * p.n_qk_heads + hq) * kD + ch * 8);
      else *reinterpret_cast<uint4*>(d) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        if (t < ns) {
          const int64_t gi = (int64_t)(t0 + c0 + t) * H + h;
          if (Rule<RULE>::kUsesGate) cp_async_4(gin + t, p.g + gi); else gin[t] = 1.0f;
          cp_async_4(gin + kC + t, p.beta + gi);
        } else {
          gin[t] = 1.0f;
          gin[kC + t] = 0.0f;
        }
      }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    // gates (warp 0): the gate block -- gamma_t, gamma_C / gamma_t, the factored ratios
    // gamma_t / gamma_s = A_t B_s around the chunk's middle, log |gamma_t|, its sign -- and b_t
    if (warp == 0) {
      float lg[2], sg[2];
      bool big = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        float a, bc, cc;
        Rule<RULE>::coeffs(gin[t], gin[kC + t], a, bc, cc);
        big |= fabsf(a) > 1.0f;
        lg[e] = __logf(fmaxf(fabsf(a), 1e-30f));
        sg[e] = a < 0.0f ? -1.0f : 1.0f;
        sBt[t] = bc;
      }
      float l = lg[0] + lg[1], sgn = sg[0] * sg[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float lo2 = __shfl_up_sync(0xffffffffu, l, off);
        const float so2 = __shfl_up_sync(0xffffffffu, sgn, off);
        if (lane >= off) {
          l += lo2;
          sgn *= so2;
        }
      }
      const float lprev = l - (lg[0] + lg[1]), sprev = sgn * sg[0] * sg[1];  // exclusive (signs are +-1)
      const float lv[2] = {lprev + lg[0], l}, sv[2] = {sprev * sg[0], sgn};
      const float lfirst = __shfl_sync(0xffffffffu, lv[0], 0), llast = __shfl_sync(0xffffffffu, l, 31);
      const float slast = __shfl_sync(0xffffffffu, sgn, 31);
      const bool fact = !__any_sync(0xffffffffu, big) && (lfirst - llast) <= 80.0f;
      const float m = 0.5f * (lfirst + llast);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        gbk[t] = sv[e] * __expf(lv[e]);
        gbk[kC + t] = slast * sv[e] * __expf(llast - lv[e]);
        gbk[2 * kC + t] = sv[e] * __expf(lv[e] - m);
        gbk[3 * kC + t] = sv[e] * __expf(m - lv[e]);
        gbk[4 * kC + t] = lv[e];
        gbk[5 * kC + t] = sv[e];
      }
      if (lane < 4) gbk[6 * kC + lane] = (lane == 0 && fact) ? 1.0f : 0.0f;
    }
    __syncthreads();
    const bool fact = gbk[6 * kC] != 0.0f;
    const float* sGm = gbk;
    const float* sFa = gbk + 2 * kC;
    const float* sFb = gbk + 3 * kC;
    const float* sLg = gbk + 4 * kC;
    const float* sSg = gbk + 5 * kC;

    // L = strictly-lower(b_t gamma_t / gamma_s k_t . k_s): warp w, rows 32 w .. + 31
    {
      float acc[2][8][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[mi][j][0] = acc[mi][j][1] = acc[mi][j][2] = acc[mi][j][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < kD; kk += 16) {
        uint32_t a0[4], a1[4];
        lda(a0, sbase + kPOffK, kRow128, 32 * warp, kk, lane);
        lda(a1, sbase + kPOffK, kRow128, 32 * warp + 16, kk, lane);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b[4];
          ldb_nk(b, sbase + kPOffK, kRow128, 16 * np, kk, lane);
          mma16816(acc[0][2 * np], a0, b[0], b[1]);
          mma16816(acc[0][2 * np + 1], a0, b[2], b[3]);
          mma16816(acc[1][2 * np], a1, b[0], b[1]);
          mma16816(acc[1][2 * np + 1], a1, b[2], b[3]);
        }
      }
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 32 * warp + 16 * mi + g8 + (e >> 1) * 8, s_ = 8 * j + 2 * t4 + (e & 1);
            float v = 0.0f;
            if (s_ < r) {
              const float ratio = fact ? sFa[r] * sFb[s_] : sSg[r] * sSg[s_] * __expf(sLg[r] - sLg[s_]);
              v = sBt[r] * ratio * acc[mi][j][e];
            }
            sL[r * kLs + s_] = v;
          }
    }
    __syncthreads();  // L complete; the K space is free for Tw, Tu

    // T = (I + L)^-1 by 32 x 32 blocks, L = [L00 0; L10 L11]:  T = [A 0; C D] with
    // A = (I + L00)^-1 (warp 0) and D = (I + L11)^-1 (warp 1) by forward substitution in
    // FP32, one column per lane (x_r = [r == c] - sum_{s < r} L_rs x_s, four partial sums),
    // then C = -D (L10 A) by both warps.  A, D and M = L10 A pass through the K space.
    {
      float* sA = reinterpret_cast<float*>(smem + kPOffK);  // [32][33] fp32
      float* sD = sA + 32 * 33;
      float* sM = sD + 32 * 33;
      const int r0 = 32 * warp;
      float x[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) x[r] = (r == lane) ? 1.0f : 0.0f;
#pragma unroll
      for (int r = 1; r < 32; ++r) {
        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
        for (int s4 = 0; s4 < r; s4 += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(sL + (r0 + r) * kLs + r0 + s4);
          a0 = fmaf(l4.x, x[s4], a0);
          if (s4 + 1 < r) a1 = fmaf(l4.y, x[s4 + 1], a1);
          if (s4 + 2 < r) a2 = fmaf(l4.z, x[s4 + 2], a2);
          if (s4 + 3 < r) a3 = fmaf(l4.w, x[s4 + 3], a3);
        }
        x[r] -= (a0 + a1) + (a2 + a3);
      }
      float* sBlk = warp == 0 ? sA : sD;
#pragma unroll
      for (int r = 0; r < 32; ++r) sBlk[r * 33 + lane] = x[r];
      __syncthreads();
      // M = L10 A: column lane, rows 16 warp .. + 15
      float acc[16];
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) acc[i2] = 0.0f;
#pragma unroll 4
      for (int k = 0; k < 32; ++k) {
        const float a = sA[k * 33 + lane];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) acc[i2] = fmaf(sL[(32 + 16 * warp + i2) * kLs + k], a, acc[i2]);
      }
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) sM[(16 * warp + i2) * 33 + lane] = acc[i2];
      __syncthreads();
      // C = -D M: column lane, rows 16 warp .. + 15
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) acc[i2] = 0.0f;
#pragma unroll 4
      for (int k = 0; k < 32; ++k) {
        const float mv = sM[k * 33 + lane];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) acc[i2] = fmaf(sD[(16 * warp + i2) * 33 + k], mv, acc[i2]);
      }
      __syncthreads();  // A, D and M are read: the K space takes Tw, Tu
      // Tw = T diag(b gamma), Tu = T diag(b) (BF16, rows 128 bytes apart, piece ^ (row & 7))
      auto put = [&](int r, int c, float v) {
        const uint32_t off = kPOffK + r * kRow64 + (((c >> 3) ^ (r & 7)) << 4) + 2 * (c & 7);
        *reinterpret_cast<__nv_bfloat16*>(smem + off) = __float2bfloat16_rn(v * sBt[c] * sGm[c]);
        *reinterpret_cast<__nv_bfloat16*>(smem + off + kC * kRow64) = __float2bfloat16_rn(v * sBt[c]);
      };
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        put(r0 + r, r0 + lane, x[r]);           // A or D
        if (warp == 1) put(r, 32 + lane, 0.0f);  // the zero block above D
      }
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) put(32 + 16 * warp + i2, lane, -acc[i2]);  // C
    }
    __syncthreads();
    // Tw, Tu and the gate block to the workspace (contiguous in shared memory as in the tile)
    uint4* dstw = reinterpret_cast<uint4*>(static_cast<unsigned char*>(const_cast<void*>(p.workspace)) + kWsHeadBytes +
                                           ((int64_t)gc * H + h) * kPrepTileBytes);
    const uint4* srcw = reinterpret_cast<const uint4*>(smem + kPOffK);
    for (int idx = tid; idx < kPrepTileBytes / 16; idx += kPThreads) dstw[idx] = srcw[idx];
    __syncthreads();
  }
}

template <int RULE>
cudaError_t launch_chunk_prep(const ScanParams& p, cudaStream_t stream) {
  const void* fn = reinterpret_cast<const void*>(&chunk_prep_kernel<RULE>);
  const int per_sm = prepare_kernel(fn, chunk::kPThreads, chunk::kPSmem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  const int64_t items = ((int64_t)(p.total_tokens + chunk::kC - 1) / chunk::kC + p.n_seqs + 1) * p.n_v_heads;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)(items < cap ? items : cap);
  if (grid <= 0) return cudaSuccess;
  chunk_prep_kernel<RULE><<<grid, chunk::kPThreads, chunk::kPSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace la
