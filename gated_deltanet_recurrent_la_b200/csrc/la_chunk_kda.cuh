// la_chunk_kda.cuh -- the chunked prefill of the channel-wise gate (rule kda) in two launches
// on the tensor cores.
//
// Algebra ("Seven Architectures Replacing KV Cache With Bounded Mutable State": the "Kimi
// Linear" section, whose transition S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} +
// beta_t k_t v_t^T admits a chunkwise-parallel evaluation, and the "Gated DeltaNet-2"
// section's chunkwise WY form).  Per (sequence, head) and chunk of C = 64 tokens, with
// Gamma_t = prod_{s <= t} alpha_s (a d_k vector) and S0 the state at the chunk start, the
// decays are absorbed into the operands:
//
//   K+ = K (.) Gamma,   Q+ = Q (.) Gamma,   K^ = K (.) Gamma_C / Gamma
//   L_ts = beta_t sum_i k_ti k_si Gamma_ti / Gamma_si  (s < t),  P_ts the same with q_t (s <= t)
//   T = (I + L)^-1,  Tw = T diag(beta),  W = Tw K+,  U = Tw V - W S0
//   O = scale (Q+ S0 + P U),   S = Diag(Gamma_C) S0 + K^^T U
//
// The ratios Gamma_ti / Gamma_si sit inside the sums over i, so they are factored: per
// 16-token block b around a reference m_b (the mean of the log-magnitudes l = log|Gamma| at
// the block's two ends), Gamma_ti / Gamma_si = E_ti F_{b(t) b(s) i} R_si with
// E_t = sigma_t e^{l_t - m_b(t)}, R_s = sigma_s e^{m_b(s) - l_s}, F_bj = e^{m_b - m_j} (<= 1 for
// b >= j when the decays are at most 1 in magnitude).  Each token's log-magnitude is held
// to [-8, 8], so E and R stay within e^{+-64}: decay magnitudes below e^-8, zero included,
// act as e^-8 (a change of at most e^-8 of a decayed state row, below the BF16 operand
// precision of the chunked form).
//
// Launch 1 (chunk_kda_prep_kernel): one (chunk, head) tile per CTA of 4 warps, two CTAs per
// SM.  The chunk's log-magnitudes and signs (one channel per thread, a running sum over
// the tokens), then per 16-byte piece the operands A = [Q; K] (.) E and B = K (.) R in
// shared memory and Q+, K+, K^ straight to the workspace tile; [Q; K] B^T by warp-level
// BF16 MMAs with F applied to the B fragments, masked into P and L; the UT inverse; Tw.
// Launch 2 (chunk_kda_kernel): the recurrence on the fifth-generation tensor cores, one
// CTA per SM, the state in tensor memory, V by TMA and the tile by one bulk copy per chunk.
#pragma once

#include <cstdint>
#include <cstring>

#include "la_chunk.cuh"
#include "la_chunk_fused.cuh"
#include "la_umma.cuh"

namespace la {
namespace kda {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr float kLogClamp = 8.0f;

// workspace tile of one (chunk, head), bytes: BF16 operands in 64-column panels (rows 128
// bytes apart, the 16-byte piece c of row r at c ^ (r & 7)), then Gamma_C
constexpr int kTileTw = 0;              // Tw = T diag(beta)  [64 t][64 s]
constexpr int kTileP = 8192;            // P                  [64 t][64 s]
constexpr int kTileQp = 16384;          // Q+   [64 t][128]: two panels of 64 rows
constexpr int kTileKp = 32768;          // K+
constexpr int kTileKh = 49152;          // K^
constexpr int kTileGc = 65536;          // Gamma_C [128] fp32
constexpr int kTileCopy = kTileGc + 512;  // bytes the recurrence copies per chunk
constexpr int kTileBytes = 66560;       // tiles 1024 bytes apart
constexpr int kWsHeadBytes = 256;

// prep launch, shared memory (bytes)
constexpr int kPThreads = 128;
constexpr int kPOffQ = 0;                         // Q, then A_Q = Q (.) E   [64][128] bf16, rows 256 B, swizzled
constexpr int kPOffK = 16384;                     // K, then A_K = K (.) E
constexpr int kPOffB = 32768;                     // B = K (.) R
constexpr int kPOffLam = 49152;                   // alpha, then l [64][128] fp32; then the Tw and P panels
constexpr int kPOffSgn = kPOffLam + 32768;        // sign bits [64 t][4 words of 32 channels]
constexpr int kPOffM = kPOffSgn + 1024;           // m_b                   [4][128] fp32
constexpr int kPOffEm = kPOffM + 2048;            // e^{m_b}               [4][128]
constexpr int kPOffCm = kPOffEm + 2048;           // sigma_C e^{l_C - m_b} [4][128]
constexpr int kPOffF = kPOffCm + 2048;            // F_bj [6][128]: (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
constexpr int kPOffL = kPOffF + 3072;             // L, then T [64][kLs] fp32
constexpr int kPOffX = kPOffL + kC * chunk::kLs * 4;
constexpr int kPOffBeta = kPOffX + 3 * 16 * chunk::kXs * 4;
constexpr int kPSmem = kPOffBeta + kC * 4;
static_assert(2 * (kPSmem + 1024) <= 228 * 1024, "two prep CTAs per SM");
static_assert(kPOffL % 16 == 0 && kPOffX % 16 == 0, "alignment");

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t w, float2 f) {
  return pack_bf16x2(bf16_lo(w) * f.x, bf16_hi(w) * f.y);
}

}  // namespace kda

// tiles of the workspace: chunk c of sequence s is tile (t0_s / 64 + s + c) (distinct for
// every chunk; fewer than T / 64 + n_seqs + 1), the (tile, head) pair at tile * H + head
inline size_t kda_workspace_bytes(int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads) {
  if (total_tokens < 0 || n_seqs < 0 || n_v_heads <= 0) return 0;
  const int64_t tiles = (total_tokens + kda::kC - 1) / kda::kC + n_seqs + 1;
  return (size_t)(kda::kWsHeadBytes + tiles * n_v_heads * kda::kTileBytes);
}

__global__ void __launch_bounds__(kda::kPThreads, 2) chunk_kda_prep_kernel(const ScanParams p) {
  using namespace kda;
  using chunk::kLs;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_addr(smem);
  float* lam = reinterpret_cast<float*>(smem + kPOffLam);
  uint32_t* sgn = reinterpret_cast<uint32_t*>(smem + kPOffSgn);
  float* sM = reinterpret_cast<float*>(smem + kPOffM);
  float* sEm = reinterpret_cast<float*>(smem + kPOffEm);
  float* sCm = reinterpret_cast<float*>(smem + kPOffCm);
  float* sF = reinterpret_cast<float*>(smem + kPOffF);
  float* sL = reinterpret_cast<float*>(smem + kPOffL);
  float* sX = reinterpret_cast<float*>(smem + kPOffX);
  float* sBeta = reinterpret_cast<float*>(smem + kPOffBeta);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int H = p.n_v_heads;
  const int ratio_h = H / p.n_qk_heads;
  if (p.n_seqs <= 0) return;
  const int64_t n_tiles = (int64_t)(p.total_tokens + kC - 1) / kC + p.n_seqs + 1;
  const int64_t items = n_tiles * H;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(p.k);
  unsigned char* ws = static_cast<unsigned char*>(const_cast<void*>(p.workspace)) + kWsHeadBytes;

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
    unsigned char* tile = ws + item * kTileBytes;

    // Q and K rows (zero beyond the sequence), the decays (1 beyond it) and beta (0 beyond it)
    for (int idx = tid; idx < kC * 16; idx += kPThreads) {
      const int r = idx >> 4, ch = idx & 15;
      const uint32_t so = chunk::swz(0u, r, ch, 256);
      if (r < ns) {
        const int64_t row = (int64_t)(t0 + c0 + r) * p.n_qk_heads + hq;
        cp_async_16(smem + kPOffQ + so, qg + row * kD + ch * 8);
        cp_async_16(smem + kPOffK + so, kg + row * kD + ch * 8);
      } else {
        *reinterpret_cast<uint4*>(smem + kPOffQ + so) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + kPOffK + so) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    for (int idx = tid; idx < kC * 32; idx += kPThreads) {
      const int r = idx >> 5, pc = idx & 31;
      if (r < ns)
        cp_async_16(lam + r * kD + 4 * pc, p.g + ((int64_t)(t0 + c0 + r) * H + h) * kD + 4 * pc);
      else
        *reinterpret_cast<float4*>(lam + r * kD + 4 * pc) = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
    }
    if (tid < kC) {
      if (tid < ns) cp_async_4(sBeta + tid, p.beta + (int64_t)(t0 + c0 + tid) * H + h);
      else sBeta[tid] = 0.0f;
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    // channel i = tid: l_t = sum_{s <= t} clamp(log |alpha_s|), the sign of Gamma_t (bits per
    // token and 32 channels), the block references m_b, and the per-channel factors
    {
      const int i = tid;
      float l = 0.0f, lstart = 0.0f;
      bool neg = false;
#pragma unroll 4
      for (int t = 0; t < kC; ++t) {
        const float a = lam[t * kD + i];
        l += fminf(fmaxf(__logf(fabsf(a)), -kLogClamp), kLogClamp);
        neg ^= (a < 0.0f);
        lam[t * kD + i] = l;
        const uint32_t bits = __ballot_sync(0xffffffffu, neg);
        if (lane == 0) sgn[t * 4 + warp] = bits;
        if ((t & 15) == 15) {
          sM[(t >> 4) * kD + i] = 0.5f * (lstart + l);
          lstart = l;
        }
      }
      const float sc = neg ? -1.0f : 1.0f;  // the sign of Gamma_C; l is l_C
      float m[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        m[b] = sM[b * kD + i];
        sEm[b * kD + i] = __expf(m[b]);
        sCm[b * kD + i] = sc * __expf(l - m[b]);
      }
      sF[0 * kD + i] = __expf(m[1] - m[0]);
      sF[1 * kD + i] = __expf(m[2] - m[0]);
      sF[2 * kD + i] = __expf(m[2] - m[1]);
      sF[3 * kD + i] = __expf(m[3] - m[0]);
      sF[4 * kD + i] = __expf(m[3] - m[1]);
      sF[5 * kD + i] = __expf(m[3] - m[2]);
      reinterpret_cast<float*>(tile + kTileGc)[i] = sc * __expf(l);
    }
    __syncthreads();

    // per 16-byte piece (token t, channels 8c .. 8c + 7): A_Q, A_K and B in place / in shared
    // memory; Q+, K+ and K^ to the tile
#pragma unroll 1
    for (int idx = tid; idx < kC * 16; idx += kPThreads) {
      const int t = idx >> 4, c = idx & 15, b = t >> 4;
      const uint32_t so = chunk::swz(0u, t, c, 256);
      const uint4 qv = *reinterpret_cast<const uint4*>(smem + kPOffQ + so);
      const uint4 kv = *reinterpret_cast<const uint4*>(smem + kPOffK + so);
      const float q[8] = {bf16_lo(qv.x), bf16_hi(qv.x), bf16_lo(qv.y), bf16_hi(qv.y),
                          bf16_lo(qv.z), bf16_hi(qv.z), bf16_lo(qv.w), bf16_hi(qv.w)};
      const float k[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                          bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
      const uint32_t sb = (sgn[t * 4 + (c >> 2)] >> (8 * (c & 3))) & 0xffu;
      const float* lp = lam + t * kD + 8 * c;
      const float* mp = sM + b * kD + 8 * c;
      const float* ep = sEm + b * kD + 8 * c;
      const float* cp = sCm + b * kD + 8 * c;
      uint32_t aq[4], ak[4], bm[4], qp[4], kp[4], kh[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        float vaq[2], vak[2], vbm[2], vqp[2], vkp[2], vkh[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int e = 2 * e2 + u;
          const float sg = ((sb >> e) & 1u) ? -1.0f : 1.0f;
          const float x = lp[e] - mp[e];
          const float E = sg * __expf(x), R = sg * __expf(-x);
          const float G = E * ep[e], Kh = R * cp[e];
          vaq[u] = q[e] * E;
          vak[u] = k[e] * E;
          vbm[u] = k[e] * R;
          vqp[u] = q[e] * G;
          vkp[u] = k[e] * G;
          vkh[u] = k[e] * Kh;
        }
        aq[e2] = pack_bf16x2(vaq[0], vaq[1]);
        ak[e2] = pack_bf16x2(vak[0], vak[1]);
        bm[e2] = pack_bf16x2(vbm[0], vbm[1]);
        qp[e2] = pack_bf16x2(vqp[0], vqp[1]);
        kp[e2] = pack_bf16x2(vkp[0], vkp[1]);
        kh[e2] = pack_bf16x2(vkh[0], vkh[1]);
      }
      *reinterpret_cast<uint4*>(smem + kPOffQ + so) = make_uint4(aq[0], aq[1], aq[2], aq[3]);
      *reinterpret_cast<uint4*>(smem + kPOffK + so) = make_uint4(ak[0], ak[1], ak[2], ak[3]);
      *reinterpret_cast<uint4*>(smem + kPOffB + so) = make_uint4(bm[0], bm[1], bm[2], bm[3]);
      const uint32_t go = umma::panel_piece(kC, t, c);
      *reinterpret_cast<uint4*>(tile + kTileQp + go) = make_uint4(qp[0], qp[1], qp[2], qp[3]);
      *reinterpret_cast<uint4*>(tile + kTileKp + go) = make_uint4(kp[0], kp[1], kp[2], kp[3]);
      *reinterpret_cast<uint4*>(tile + kTileKh + go) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
    }
    __syncthreads();
    // the Tw and P panels (in the space of l): their blocks above the diagonal stay zero
    unsigned char* sTw = smem + kPOffLam;
    unsigned char* sP = smem + kPOffLam + 8192;
    for (int idx = tid; idx < 1024; idx += kPThreads)
      reinterpret_cast<uint4*>(sTw)[idx] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    // [Q; K] B^T by 16 x 16 blocks (row block b, column block j <= b), F_bj on the B
    // fragments; warp w takes rows of Q (even w) or K (odd w) of blocks {3, 0} (w < 2) or
    // {2, 1} (w >= 2): five blocks each.  Q rows give P (s <= t), K rows give L (s < t, times
    // beta_t).
    {
      const bool is_k = (warp & 1) != 0;
      const uint32_t abase = sbase + (is_k ? kPOffK : kPOffQ);
#pragma unroll 1
      for (int bsel = 0; bsel < 2; ++bsel) {
        const int b = (warp < 2) ? (bsel == 0 ? 3 : 0) : (bsel == 0 ? 2 : 1);
#pragma unroll 1
        for (int j = 0; j <= b; ++j) {
          float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          const float* F = sF + ((b * (b - 1)) / 2 + j) * kD;
#pragma unroll
          for (int kk = 0; kk < kD; kk += 16) {
            uint32_t a[4], bf[4];
            chunk::lda(a, abase, 256, 16 * b, kk, lane);
            chunk::ldb_nk(bf, sbase + kPOffB, 256, 16 * j, kk, lane);
            if (j < b) {
              const float2 f0 = *reinterpret_cast<const float2*>(F + kk + 2 * t4);
              const float2 f1 = *reinterpret_cast<const float2*>(F + kk + 8 + 2 * t4);
              bf[0] = scale_bf16x2(bf[0], f0);
              bf[1] = scale_bf16x2(bf[1], f1);
              bf[2] = scale_bf16x2(bf[2], f0);
              bf[3] = scale_bf16x2(bf[3], f1);
            }
            chunk::mma16816(acc[0], a, bf[0], bf[1]);
            chunk::mma16816(acc[1], a, bf[2], bf[3]);
          }
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int s0 = 16 * j + 8 * nt + 2 * t4;
#pragma unroll
            for (int hrow = 0; hrow < 2; ++hrow) {
              const int r = 16 * b + g8 + 8 * hrow;
              const float v0 = acc[nt][2 * hrow], v1 = acc[nt][2 * hrow + 1];
              if (!is_k) {
                *reinterpret_cast<uint32_t*>(sP + umma::panel_off(kC, r, s0)) =
                    pack_bf16x2(s0 <= r ? v0 : 0.0f, s0 + 1 <= r ? v1 : 0.0f);
              } else {
                const float bt = sBeta[r];
                *reinterpret_cast<float2*>(sL + r * kLs + s0) =
                    make_float2(s0 < r ? bt * v0 : 0.0f, s0 + 1 < r ? bt * v1 : 0.0f);
              }
            }
          }
        }
      }
    }
    __syncthreads();
    chunk::ut_inverse64(sL, sX, warp, lane, 1);
    // Tw = T diag(beta), the ten lower 16 x 16 blocks: thread tid -> row tid / 8, columns
    // 2 (tid % 8) + {0, 1} of each
    {
      const int rb = tid >> 3, cpair = 2 * (tid & 7);
#pragma unroll 2
      for (int i = 0; i < 10; ++i) {
        const int bi = i >= 6 ? 3 : i >= 3 ? 2 : i >= 1 ? 1 : 0;
        const int bj = i - (bi * (bi + 1)) / 2;
        const int row = 16 * bi + rb, col = 16 * bj + cpair;
        const float2 tv = *reinterpret_cast<const float2*>(sL + row * kLs + col);
        *reinterpret_cast<uint32_t*>(sTw + umma::panel_off(kC, row, col)) =
            pack_bf16x2(tv.x * sBeta[col], tv.y * sBeta[col + 1]);
      }
    }
    __syncthreads();
    // Tw and P to the tile (kTileTw, kTileP: the same order as in shared memory)
    for (int idx = tid; idx < 1024; idx += kPThreads)
      reinterpret_cast<uint4*>(tile + kTileTw)[idx] = reinterpret_cast<const uint4*>(sTw)[idx];
    __syncthreads();  // shared memory is reused by the next tile
  }
}

// ---- launch 2: the recurrence ------------------------------------------------------------
// One CTA of 10 warps per SM walks (sequence, head) units (boustrophedon over seq_order):
//   warp 0      loads a chunk into one of two stages: V (two 64 x 64 panels) by TMA and the
//               chunk's workspace tile (Tw, P, Q+, K+, K^, Gamma_C) by one bulk copy
//   warp 1      lane 0 issues every MMA and owns the tensor-memory allocation
//   warps 2-5   the state: S0^T -> BF16 copy and S^T (.)= Gamma_C per chunk, U^T -> BF16,
//               initial and final states
//   warps 6-9   W^T -> shared memory, outputs (staged, written as 16-byte pieces)
// Per chunk: W^T = K+^T Tw^T and U^T = V^T Tw^T; U^T -= S0^T W^T; O^T = S0^T Q+^T; then
// S^T += U^T K^ and O^T += U^T P^T.  Waits as in the one-launch kernel: time limit, CTA-wide
// abort flag, MMAs and copies drained before the tensor memory is released.
namespace kda {
constexpr int kStages = 2;
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpState = 2, kWarpOut = 6;
constexpr int kThreads = 10 * 32;
constexpr uint32_t kNbState = 2, kNbOut = 3;
constexpr int kOffV = 0;                           // in a stage: V, two panels of 64 rows
constexpr int kOffTile = 16384;                    //             the workspace tile
constexpr int kStageBytes = kOffTile + kTileBytes;
constexpr int kOffWt = kStages * kStageBytes;      // W^T [128 d_k][64 t]; the outputs' staging tile
constexpr int kOffBar = kOffWt + 16384;
enum Bar {
  kFull = 0,   // [2] stage loaded (TMA and bulk-copy bytes)
  kEmpty = 2,  // [2] stage free (MMA commit)
  kWFull = 4,  // W^T and U~^T in tensor memory (MMA commit)
  kWFree,      // W^T is in shared memory
  kSPass,      // S0^T copied to BF16 and S^T scaled by Gamma_C
  kUFull,      // U^T in tensor memory (MMA commit)
  kUDone,      // U^T copied to BF16
  kSFull,      // state update done (MMA commit)
  kOFull,      // outputs of a chunk in tensor memory (MMA commit)
  kOFree,      // outputs read
  kDrain,      // every MMA issued has completed
  kNumBars
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // [0] tensor-memory base, [1] abort
constexpr int kSmem = kOffMisc + 16 + 1024;       // + slack for the 1024-byte alignment
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kStageBytes % 1024 == 0 && kOffWt % 1024 == 0 && kTileCopy % 16 == 0, "alignment");
constexpr uint32_t kStageTx = 16384 + kTileCopy;  // bytes landing in a stage per chunk

constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0;     // S^T        [d_v][d_k]     128
constexpr int kColSb = 128;  // S0^T BF16  [d_v][d_k / 2]  64 (A operand)
constexpr int kColW = 192;   // W^T        [d_k][64]       64
constexpr int kColU = 256;   // U^T        [d_v][64]       64
constexpr int kColUb = 320;  // U^T BF16   [d_v][32]       32 (A operand)
constexpr int kColO = 384;   // O^T        [d_v][64]       64
}  // namespace kda

__global__ void __launch_bounds__(kda::kThreads, 1) chunk_kda_kernel(const ScanParams p,
                                                                   const __grid_constant__ TcMaps maps) {
  using namespace kda;
  using fused::fwait;
  using fused::gwait;
  using fused::mma_ts;
  using fused::pack2;
  using fused::Unit;
  using fused::unit_info;
  using fused::unit_of;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = misc + 1;
  const unsigned char* ws = static_cast<const unsigned char*>(p.workspace) + kWsHeadBytes;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int H = p.n_v_heads;
  const int64_t units = (int64_t)p.n_seqs * H;
  const int64_t G = gridDim.x;

  if (warp == kWarpMma) umma::alloc(const_cast<uint32_t*>(misc), kTmemCols);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kFull + s], 1);
      mbar_init(&bars[kEmpty + s], 1);
    }
    for (int b = kWFull; b < kNumBars; ++b) mbar_init(&bars[b], 1);
    misc[1] = 0u;
    mbar_init_fence();
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = misc[0];

  // chunks this CTA processes (every role walks the same units in the same order)
  int64_t n_total = 0;
  for (int64_t r = 0; r * G < units; ++r) {
    const int64_t u = unit_of(r, G, blockIdx.x);
    if (u >= units) continue;
    const Unit x = unit_info(p, u);
    if (x.valid) n_total += (x.n_tok + kC - 1) / kC;
  }

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ loader
    int64_t j = 0;
    bool ok = true;
    if (lane == 0) {
      for (int64_t r = 0; ok && r * G < units; ++r) {
        const int64_t u = unit_of(r, G, blockIdx.x);
        if (u >= units) continue;
        const Unit x = unit_info(p, u);
        if (!x.valid) continue;
        const int nch = (x.n_tok + kC - 1) / kC;
        for (int c = 0; c < nch; ++c, ++j) {
          const int s = (int)(j % kStages);
          if (j >= kStages && !(ok = fwait(&bars[kEmpty + s], (uint32_t)((j / kStages) + 1) & 1u, abort_flag)))
            break;
          unsigned char* st = smem + s * kStageBytes;
          uint64_t* full = &bars[kFull + s];
          const int64_t gtile = (int64_t)(x.t0 / kC + x.seq + c) * H + x.h;
          mbar_arrive_expect_tx(full, kStageTx);
          umma::tma_load_3d(st + kOffV, &maps.v, 0, x.h, x.t0 + c * kC, full);
          umma::tma_load_3d(st + kOffV + 8192, &maps.v, 64, x.h, x.t0 + c * kC, full);
          bulk_g2s(st + kOffTile, ws + gtile * kTileBytes, (uint32_t)kTileCopy, full);
        }
      }
      // copies still in flight (after an abort): let them land, within the limit
      for (int64_t jj = (j > kStages ? j - kStages : 0); jj < j; ++jj)
        mbar_wait(&bars[kFull + (int)(jj % kStages)], (uint32_t)(jj / kStages) & 1u);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdMK64 = umma::idesc_bf16(128, 64, true, false);         // A MN-major
      constexpr uint32_t kIdTM64n = umma::idesc_bf16(128, 64, false, true, true);  // A tmem, B MN, -A
      constexpr uint32_t kIdTK64 = umma::idesc_bf16(128, 64, false, false);        // A tmem, B K-major
      constexpr uint32_t kIdTM128 = umma::idesc_bf16(128, 128, false, true);       // A tmem, B MN-major
      const uint64_t dWm = umma::sdesc(sb + kOffWt, 16384, 1024);
      auto W = [&](int b, int64_t ph) { return fwait(&bars[b], (uint32_t)ph & 1u, abort_flag); };
      bool ok = true;
      for (int64_t j = 0; ok && j < n_total; ++j) {
        const int s = (int)(j % kStages);
        const uint32_t st = sb + (uint32_t)s * kStageBytes;
        const uint32_t tl = st + kOffTile;
        const uint64_t dVm = umma::sdesc(st + kOffV, 8192, 1024);     // V as MN-major (M = d_v)
        const uint64_t dTw = umma::sdesc(tl + kTileTw, 16, 1024);    // Tw rows, K-major
        const uint64_t dP = umma::sdesc(tl + kTileP, 16, 1024);      // P rows, K-major
        const uint64_t dQp = umma::sdesc(tl + kTileQp, 16, 1024);    // Q+ rows, K-major (K = d_k)
        const uint64_t dKp = umma::sdesc(tl + kTileKp, 8192, 1024);  // K+ as MN-major (M = d_k)
        const uint64_t dKh = umma::sdesc(tl + kTileKh, 8192, 1024);  // K^ as MN-major (N = d_k)
        if (!(ok = W(kFull + s, j / kStages))) break;
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // W^T = K+^T Tw^T (K = tokens)
          umma::mma(tmem + kColW, umma::sdesc_add(dKp, kk * 2048), umma::sdesc_add(dTw, kk * 32), kIdMK64, kk);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // U^T = V^T Tw^T
          umma::mma(tmem + kColU, umma::sdesc_add(dVm, kk * 2048), umma::sdesc_add(dTw, kk * 32), kIdMK64, kk);
        umma::commit(&bars[kWFull]);
        if (!(ok = W(kWFree, j) && W(kSPass, j))) break;
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // U^T -= S0^T W^T (K = d_k)
          mma_ts(tmem + kColU, tmem + kColSb + 8 * kk, umma::sdesc_add(dWm, kk * 2048), kIdTM64n, 1);
        umma::commit(&bars[kUFull]);
        if (j > 0 && !(ok = W(kOFree, j - 1))) break;
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // O^T = S0^T Q+^T (K = d_k)
          const uint32_t ko = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_ts(tmem + kColO, tmem + kColSb + 8 * kk, umma::sdesc_add(dQp, ko), kIdTK64, kk);
        }
        if (!(ok = W(kUDone, j))) break;
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // S^T += U^T K^ (K = tokens)
          mma_ts(tmem + kColS, tmem + kColUb + 8 * kk, umma::sdesc_add(dKh, kk * 2048), kIdTM128, 1);
        umma::commit(&bars[kSFull]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // O^T += U^T P^T
          mma_ts(tmem + kColO, tmem + kColUb + 8 * kk, umma::sdesc_add(dP, kk * 32), kIdTK64, 1);
        umma::commit(&bars[kOFull]);
        umma::commit(&bars[kEmpty + s]);
      }
      // every MMA issued completes before the tensor memory is released
      umma::commit(&bars[kDrain]);
      mbar_wait(&bars[kDrain], 0);
    }
  } else if (warp < kWarpOut) {
    // ------------------------------------------------------------------ state group
    const int tp = tid - kWarpState * 32;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // d_v index
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
    int64_t j = 0;
    bool ok = true;
    for (int64_t ru = 0; ok && ru * G < units; ++ru) {
      const int64_t u = unit_of(ru, G, blockIdx.x);
      if (u >= units) continue;
      const Unit x = unit_info(p, u);
      if (x.err && tp == 0) report(p.err, x.err);
      if (!x.valid) continue;
      const int nch = (x.n_tok + kC - 1) / kC;
      const int64_t sbase_src = ((int64_t)x.rs * H + x.h) * (kD * kD);
      const int64_t dbase = ((int64_t)x.ws * H + x.h) * (kD * kD);
      auto store_col = [&](int64_t base, int i0, const uint32_t* v) {  // S[i0 + e][r] = v[e], e < 16
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int64_t el = base + (int64_t)(i0 + e) * kD + r;
          if (p.dst_dtype == LA_F32)
            static_cast<float*>(p.dst)[el] = __uint_as_float(v[e]);
          else
            static_cast<__nv_bfloat16*>(p.dst)[el] = __float2bfloat16_rn(__uint_as_float(v[e]));
        }
      };
      if (nch == 0) {
        // empty sequence: the initial state (or zero) goes to the destination
        for (int i = 0; i < kD; ++i) {
          float v = 0.0f;
          if (p.read_slot)
            v = p.src_dtype == LA_F32 ? static_cast<const float*>(p.src)[sbase_src + i * kD + r]
                                      : __bfloat162float(static_cast<const __nv_bfloat16*>(p.src)[sbase_src + i * kD + r]);
          if (p.dst_dtype == LA_F32)
            static_cast<float*>(p.dst)[dbase + i * kD + r] = v;
          else
            static_cast<__nv_bfloat16*>(p.dst)[dbase + i * kD + r] = __float2bfloat16_rn(v);
        }
        continue;
      }
      // initial state S^T: lane = d_v index r, columns = d_k
#pragma unroll 1
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = 16 * c16 + e;
          float sv = 0.0f;
          if (p.read_slot) {
            const int64_t el = sbase_src + (int64_t)i * kD + r;
            sv = p.src_dtype == LA_F32 ? static_cast<const float*>(p.src)[el]
                                       : __bfloat162float(static_cast<const __nv_bfloat16*>(p.src)[el]);
          }
          v[e] = __float_as_uint(sv);
        }
        umma::st16(tq + kColS + 16 * c16, v);
      }
      umma::wait_st();
      for (int c = 0; c < nch; ++c, ++j) {
        const int s = (int)(j % kStages);
        const float* gcv = reinterpret_cast<const float*>(smem + s * kStageBytes + kOffTile + kTileGc);
        // the previous chunk's state update and this chunk's tile (the stage is not reloaded
        // before this chunk's last MMA, which waits for this group)
        if (tp == 0) {
          if (c > 0) ok = fwait(&bars[kSFull], (uint32_t)(j - 1) & 1u, abort_flag);
          if (ok) ok = fwait(&bars[kFull + s], (uint32_t)(j / kStages) & 1u, abort_flag);
        }
        if (named_bar_or(kNbState, 128, !ok)) {
          ok = false;
          break;
        }
        umma::fence_after();
        // S pass: S0^T -> BF16 (the A operand of this chunk's products), S^T[r][i] *= Gamma_C[i]
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          uint32_t a[16], b[16], w[16];
          umma::ld16(tq + kColS + 32 * c32, a);
          umma::ld16(tq + kColS + 32 * c32 + 16, b);
          umma::wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w[e] = pack2(a[2 * e], a[2 * e + 1]);
            w[8 + e] = pack2(b[2 * e], b[2 * e + 1]);
          }
          umma::st16(tq + kColSb + 16 * c32, w);
          const float* gq = gcv + 32 * c32;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            a[e] = __float_as_uint(__uint_as_float(a[e]) * gq[e]);
            b[e] = __float_as_uint(__uint_as_float(b[e]) * gq[16 + e]);
          }
          umma::st16(tq + kColS + 32 * c32, a);
          umma::st16(tq + kColS + 32 * c32 + 16, b);
        }
        umma::wait_st();
        umma::fence_before();
        named_bar_sync(kNbState, 128);
        if (tp == 0) mbar_arrive(&bars[kSPass]);
        if (!(ok = gwait(&bars[kUFull], (uint32_t)j & 1u, abort_flag, tp, kNbState))) break;
        umma::fence_after();
        // U^T -> BF16 (the A operand of S^T += U^T K^ and O^T += U^T P^T)
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
          uint32_t a[16], b[16], w[16];
          umma::ld16(tq + kColU + 32 * c32, a);
          umma::ld16(tq + kColU + 32 * c32 + 16, b);
          umma::wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w[e] = pack2(a[2 * e], a[2 * e + 1]);
            w[8 + e] = pack2(b[2 * e], b[2 * e + 1]);
          }
          umma::st16(tq + kColUb + 16 * c32, w);
        }
        umma::wait_st();
        umma::fence_before();
        named_bar_sync(kNbState, 128);
        if (tp == 0) mbar_arrive(&bars[kUDone]);
      }
      if (!ok) break;
      // final state S[i][r] = S^T[r][i]
      if (!(ok = gwait(&bars[kSFull], (uint32_t)(j - 1) & 1u, abort_flag, tp, kNbState))) break;
      umma::fence_after();
#pragma unroll 1
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t v[16];
        umma::ld16(tq + kColS + 16 * c16, v);
        umma::wait_ld();
        store_col(dbase, 16 * c16, v);
      }
      umma::fence_before();
    }
  } else {
    // ------------------------------------------------------------------ output group
    const int tp = tid - kWarpOut * 32;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // d_k index (W^T) / d_v index (O^T)
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
    __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o);
    __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(smem + kOffWt);
    int64_t j = 0;
    bool ok = true;
    for (int64_t ru = 0; ok && ru * G < units; ++ru) {
      const int64_t u = unit_of(ru, G, blockIdx.x);
      if (u >= units) continue;
      const Unit x = unit_info(p, u);
      if (!x.valid) continue;
      const int nch = (x.n_tok + kC - 1) / kC;
      for (int c = 0; c < nch; ++c, ++j) {
        // W^T rows (lane = d_k index) -> shared memory, the B operand of the U update
        if (!(ok = gwait(&bars[kWFull], (uint32_t)j & 1u, abort_flag, tp, kNbOut))) break;
        umma::fence_after();
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
          uint32_t v[32];
          umma::ld16(tq + kColW + 32 * c32, v);
          umma::ld16(tq + kColW + 32 * c32 + 16, v + 16);
          umma::wait_ld();
#pragma unroll
          for (int pc = 0; pc < 4; ++pc)
            *reinterpret_cast<uint4*>(smem + kOffWt + umma::panel_piece(128, r, 4 * c32 + pc)) =
                make_uint4(pack2(v[8 * pc], v[8 * pc + 1]), pack2(v[8 * pc + 2], v[8 * pc + 3]),
                           pack2(v[8 * pc + 4], v[8 * pc + 5]), pack2(v[8 * pc + 6], v[8 * pc + 7]));
        }
        umma::fence_smem();
        umma::fence_before();
        named_bar_sync(kNbOut, 128);
        if (tp == 0) mbar_arrive(&bars[kWFree]);
        // outputs o_t[r] = scale O^T[r][t]: staged as a row-major [64][128] BF16 tile in the
        // W^T buffer (free: U_j, its reader, has completed), then written as 16-byte pieces
        if (!(ok = gwait(&bars[kOFull], (uint32_t)j & 1u, abort_flag, tp, kNbOut))) break;
        umma::fence_after();
#pragma unroll 1
        for (int c16 = 0; c16 < 4; ++c16) {
          uint32_t v[16];
          umma::ld16(tq + kColO + 16 * c16, v);
          umma::wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) so[(16 * c16 + e) * kD + r] = __float2bfloat16_rn(p.scale * __uint_as_float(v[e]));
        }
        umma::fence_before();
        named_bar_sync(kNbOut, 128);
        if (tp == 0) mbar_arrive(&bars[kOFree]);
        {
          const int tok0 = x.t0 + c * kC;
          const int nv = min(kC, x.n_tok - c * kC);
#pragma unroll 2
          for (int i = 0; i < 8; ++i) {
            const int idx = tp + 128 * i;
            const int t = idx >> 4, ch = idx & 15;
            if (t < nv)
              *reinterpret_cast<uint4*>(og + ((int64_t)(tok0 + t) * H + x.h) * kD + ch * 8) =
                  *reinterpret_cast<const uint4*>(so + t * kD + ch * 8);
          }
        }
        named_bar_sync(kNbOut, 128);  // the staging tile is read before the next W^T lands there
      }
    }
  }

  if (tid == 0 && *abort_flag) report(p.err, LA_DEVERR_TIMEOUT);
  umma::fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    umma::fence_after();
    umma::dealloc(tmem, kTmemCols);
  }
}

// Both launches on the stream: the intra-chunk tiles of every chunk, then the recurrence.
inline cudaError_t launch_chunk_kda(const ScanParams& p, cudaStream_t stream) {
  if (p.n_seqs <= 0) return cudaSuccess;
  const void* fp = reinterpret_cast<const void*>(&chunk_kda_prep_kernel);
  const int per_sm = prepare_kernel(fp, kda::kPThreads, kda::kPSmem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  chunk_kda_prep_kernel<<<device_sm_count() * per_sm, kda::kPThreads, kda::kPSmem, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const void* fr = reinterpret_cast<const void*>(&chunk_kda_kernel);
  // one CTA per SM: the kernel holds all of the SM's tensor memory
  if (prepare_kernel(fr, kda::kThreads, kda::kSmem) != 1) return cudaErrorInvalidConfiguration;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));  // no tokens: nothing is staged, the map is never read
  if (p.total_tokens > 0 && !encode_rows_map(&maps.v, p.v, p.n_v_heads, p.total_tokens)) return cudaErrorInvalidValue;
  const int64_t units = (int64_t)p.n_seqs * p.n_v_heads;
  const int64_t cap = device_sm_count();
  const int grid = (int)(units < cap ? units : cap);
  chunk_kda_kernel<<<grid, kda::kThreads, kda::kSmem, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace la
