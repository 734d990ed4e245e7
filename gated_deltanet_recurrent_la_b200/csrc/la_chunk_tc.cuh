// la_chunk_tc.cuh -- the recurrence of the two-launch chunked prefill on the
// fifth-generation tensor cores (tcgen05), for the delta rules.
//
// Same algebra as la_chunk.cuh ("Seven Architectures Replacing KV Cache With Bounded
// Mutable State": the "Kimi Linear" section's chunkwise-parallel kernel and the "Gated
// DeltaNet-2" section's chunkwise WY algorithm).  chunk_prep_kernel has already written
// Tw = T diag(b gamma), Tu = T diag(b) and the chunk's gate quantities (gamma_t,
// gamma_C / gamma_t, the ratio factors) of every 64-token chunk to the workspace; per
// chunk this kernel forms
//
//   P   = (Q K^T) (.) M                         M_ts = gamma_t / gamma_s, s <= t
//   U^T = V^T Tu^T - S0^T W^T,   W^T = K^T Tw^T
//   O^T = scale ( S0^T Q^T diag(gamma) + U^T P^T )
//   S^T = gamma_C S0^T + Us^T K,  Us = diag(gamma_C / gamma) U
//
// with every product an M = 128 tcgen05 MMA (M runs over d_v, d_k or the stacked rows of
// Q and K), BF16 operands from shared memory and FP32 accumulators in tensor memory.  The
// transposed forms put one d_v (or d_k) index in each tensor-memory lane, so the thread
// that owns a lane writes whole operand rows back to shared memory.  The master state
// S^T (d_v lanes x d_k columns, FP32) stays in tensor memory for the whole sequence.
//
// One CTA of 9 warps per SM: worker warp w < 8 reads tensor-memory lanes 32 (w % 4) .. + 31
// and the column half w / 4 of each accumulator; lane 0 of warp 8 only issues the MMAs and
// the TMA copies, so issuing never holds up an epilogue.  Per chunk the state-free
// products (P, W^T, U~) are issued as soon as the chunk has landed and run beside the S
// pass; O1 follows it; the U update, then the state update and O2.  Four mbarriers signal
// MMA completion (P and W^T; U; the state; O2) and two the staged chunks; every wait gives
// up after a time limit (LA_DEVERR_TIMEOUT).  A chunk's outputs are assembled during the
// next chunk.  (Sequence, head) units come from a counter in the workspace header.
#pragma once

#include <cstdint>
#include <cstring>

#include "la_chunk.cuh"
#include "la_umma.cuh"

namespace la {
namespace chunk_tc {

constexpr int kC = 64;   // tokens per chunk
constexpr int kD = 128;  // d_k = d_v
constexpr int kWorkers = 256;             // 8 warps: tensor-memory epilogues, staging
constexpr int kThreads = kWorkers + 32;   // + 1 warp whose lane 0 issues the MMAs

// shared memory (bytes from a 1024-byte aligned base); operands in 64-column panels
constexpr int kBufBytes = 67584;             // one staged chunk:
constexpr int kOffQK = 0;                    //   Q rows 0..63 and K rows 64..127, [128][128]
constexpr int kOffV = 32768;                 //   V [64][128]
constexpr int kOffTw = 49152;                //   Tw [64][64]       } the workspace tile
constexpr int kOffTu = 57344;                //   Tu [64][64]       }
constexpr int kOffGB = 65536;                //   gate block        }
constexpr int kOffS = 2 * kBufBytes;         // S0^T  [128 d_v][128 d_k] BF16
constexpr int kOffW = kOffS + 32768;         // W^T   [128 d_k][64]
constexpr int kOffP = kOffW + 16384;         // P     [64][64]
constexpr int kOffU = kOffP + 8192;          // U^T   [128 d_v][64]; O [64][128] row-major at the end
constexpr int kOffUs = kOffU + 16384;        // Us^T  [128 d_v][64]
constexpr int kOffGo = kOffUs + 16384;       // gamma_t of the last two chunks [2][64] fp32 (outputs)
constexpr int kOffBar = kOffGo + 2 * kC * 4; // MMA groups 1-3, the two staging buffers, O2, drain
constexpr int kOffMisc = kOffBar + 7 * 8;    // [0] tensor-memory base, [3] the next unit
constexpr int kSmem = kOffMisc + 16 + 1024;  // + slack for the 1024-byte alignment
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(chunk::kPrepTileBytes == 16384 + chunk::kGateBlockBytes && kOffTu == kOffTw + 8192 &&
                  kOffGB == kOffTu + 8192 && kOffGB + chunk::kGateBlockBytes <= kBufBytes && kBufBytes % 1024 == 0,
              "workspace tile = Tw, Tu, gate block");

// tensor-memory columns (FP32 accumulators, 128 lanes each)
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0;     // S^T   128 columns (d_k)
constexpr int kColP = 128;   // [Q; K] K^T, 64 columns (lanes 0..63 are Q K^T)
constexpr int kColW = 192;   // W^T   64
constexpr int kColU = 256;   // U^T   64
constexpr int kColO1 = 320;  // S0^T Q^T   2 x 64 (chunk parity: read back during the next chunk)
constexpr int kColO2 = 448;  // U^T P^T    64

__device__ __forceinline__ uint4 pack8(const uint32_t* r) {
  return make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                    pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                    pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                    pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
}

// bytes that land in a staging buffer per chunk: Q, K, V (two 64 x 64 panels each) and
// the workspace tile
constexpr uint32_t kStageBytes = 6 * kC * 128 + chunk::kPrepTileBytes;

}  // namespace chunk_tc

// Tensor maps of q, k and v, each [tokens][heads][128] BF16 viewed as the 3-D array
// {128, heads, tokens}; box {64, 1, 64} with the 128-byte swizzle, i.e. one 64 x 64 panel.
struct TcMaps {
  CUtensorMap q, k, v;
};

template <int RULE>
__global__ void __launch_bounds__(chunk_tc::kThreads, 1) chunk_tc_kernel(const ScanParams p,
                                                                         const __grid_constant__ TcMaps maps) {
  using namespace chunk_tc;
  static_assert(Rule<RULE>::kPredicts, "the delta rules only");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);

  constexpr bool kGate = Rule<RULE>::kUsesGate;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool worker = warp < 8;
  const int q4 = warp & 3;         // tensor-memory lane quarter
  const int hf = (warp >> 2) & 1;  // column half
  const int lrow = 32 * q4 + lane; // this thread's lane: a d_v (or d_k, or token) index
  const int H = p.n_v_heads;
  const int ratio_h = H / p.n_qk_heads;
  const int64_t units = (int64_t)p.n_seqs * H;
  __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o);

  if (warp == 0) umma::alloc(const_cast<uint32_t*>(misc), kTmemCols);
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    mbar_init(&bars[3], 1);
    mbar_init(&bars[4], 1);
    mbar_init(&bars[5], 1);
    mbar_init(&bars[6], 1);
    mbar_init_fence();
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);  // this warp's lane quarter
  uint32_t phase = 0;   // chunks completed by this CTA: the parity of the MMA-group barriers
  uint32_t lpar = 0;    // bit b: the parity of staging buffer b's next completion
  uint32_t pending = 0; // bit b: staging buffer b has copies in flight (issuer lane)
  bool abort = false;

  // instruction descriptors
  constexpr uint32_t kIdKK64 = umma::idesc_bf16(128, 64, false, false);
  constexpr uint32_t kIdMK64 = umma::idesc_bf16(128, 64, true, false);
  constexpr uint32_t kIdKM64n = umma::idesc_bf16(128, 64, false, true, true);
  constexpr uint32_t kIdKM128 = umma::idesc_bf16(128, 128, false, true);

  // units are handed out one at a time from the workspace's counter (zeroed by the prep
  // launch), in seq_order order: longest sequences first, each CTA taking the next unit
  // when it finishes one
  unsigned int* next_unit = static_cast<unsigned int*>(const_cast<void*>(p.workspace));
#pragma unroll 1
  for (;;) {
    if (tid == 0) misc[3] = atomicAdd(next_unit, 1u);
    __syncthreads();
    const int64_t u = misc[3];
    __syncthreads();  // (misc[3] is rewritten at the next unit)
    if (u >= units) break;
    const int64_t si = u / H;
    const int h = (int)(u % H);
    const int hq = h / ratio_h;
    const int seq = p.seq_order ? __ldg(p.seq_order + si) : (int)si;
    if (seq < 0 || seq >= p.n_seqs) {
      if (tid == 0) report(p.err, LA_DEVERR_CU_SEQLENS);
      continue;
    }
    const int t0 = __ldg(p.cu_seqlens + seq);
    const int t1 = __ldg(p.cu_seqlens + seq + 1);
    if (seq == 0 && h == 0 && t0 != 0 && tid == 0) report(p.err, LA_DEVERR_CU_SEQLENS);
    if (t0 < 0 || t1 < t0 || t1 > p.total_tokens) {
      if (tid == 0) report(p.err, LA_DEVERR_CU_SEQLENS);
      continue;
    }
    const int rs = p.read_slot ? __ldg(p.read_slot + seq) : 0;
    const int ws = p.write_slot ? __ldg(p.write_slot + seq) : seq;
    const bool rs_ok = !p.read_slot || (rs >= 0 && rs < p.src_slots);
    const bool ws_ok = ws >= 0 && ws < p.dst_slots;
    if (!rs_ok || !ws_ok) {
      if (tid == 0) report(p.err, (rs_ok ? 0u : LA_DEVERR_READ_SLOT) | (ws_ok ? 0u : LA_DEVERR_WRITE_SLOT));
      continue;
    }

    // ---- initial state S^T into tensor memory: lane = d_v index, columns = d_k (64 per half)
    const int64_t sbase_src = ((int64_t)rs * H + h) * (kD * kD);
#pragma unroll 1
    for (int c16 = 0; c16 < (worker ? 4 : 0); ++c16) {
      uint32_t r[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int i = 64 * hf + 16 * c16 + x;
        float s = 0.0f;
        if (p.read_slot) {
          const int64_t e = sbase_src + (int64_t)i * kD + lrow;
          s = p.src_dtype == LA_F32 ? static_cast<const float*>(p.src)[e]
                                    : __bfloat162float(static_cast<const __nv_bfloat16*>(p.src)[e]);
        }
        r[x] = __float_as_uint(s);
      }
      umma::st16(tq + kColS + 64 * hf + 16 * c16, r);
    }
    if (worker) umma::wait_st();

    const int n_tok = t1 - t0;
    const int n_chunks = (n_tok + kC - 1) / kC;

    // Stages chunk ci into buffer ci & 1 with the TMA engine (the issuer lane): the Q, K and
    // V panels by tensor maps (rows beyond the last token read as zero) and the workspace
    // tile (Tw, Tu, gate block) as one bulk copy; all of it completes on bars[3 + (ci & 1)].
    auto stage = [&](int ci) {
      if (tid != kWorkers) return;
      const int b = ci & 1;
      unsigned char* buf = smem + b * kBufBytes;
      const int tok0 = t0 + ci * kC;
      uint64_t* full = &bars[3 + b];
      mbar_arrive_expect_tx(full, kStageBytes);
#pragma unroll
      for (int pnl = 0; pnl < 2; ++pnl) {
        umma::tma_load_3d(buf + kOffQK + pnl * 16384, &maps.q, 64 * pnl, hq, tok0, full);
        umma::tma_load_3d(buf + kOffQK + pnl * 16384 + kC * 128, &maps.k, 64 * pnl, hq, tok0, full);
        umma::tma_load_3d(buf + kOffV + pnl * 8192, &maps.v, 64 * pnl, h, tok0, full);
      }
      bulk_g2s(buf + kOffTw,
               static_cast<const unsigned char*>(p.workspace) +
                   chunk::kWsHeadBytes + (((int64_t)(tok0 / kC + seq)) * H + h) * chunk::kPrepTileBytes,
               chunk::kPrepTileBytes, full);
      pending |= 1u << b;
    };

    // The outputs of chunk cj: o_t[j] = scale (gamma_t O1^T[j][t] + O2^T[j][t]), lane = j,
    // into the U space as a row-major [64][128] BF16 tile (o_tile), then its rows to o,
    // 256 contiguous bytes per token (o_rows).  Both run one chunk late, beside the next
    // chunk's first two MMA groups on the tensor cores.
    __nv_bfloat16* sO = reinterpret_cast<__nv_bfloat16*>(smem + kOffU);
    auto o_tile = [&](int cj) -> bool {
      if (!worker) return true;
      // O2 of chunk cj (committed at the end of chunk cj, the CTA's chunk number phase - 1)
      const bool okw = mbar_wait(&bars[5], (phase - 1u) & 1u);
      umma::fence_after();
      const float* gm = reinterpret_cast<const float*>(smem + kOffGo) + (cj & 1) * kC;
#pragma unroll
      for (int c16 = 0; c16 < 2; ++c16) {
        uint32_t r1[16], r2[16];
        umma::ld16(tq + kColO1 + 64 * (cj & 1) + 32 * hf + 16 * c16, r1);
        umma::ld16(tq + kColO2 + 32 * hf + 16 * c16, r2);
        umma::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int t = 32 * hf + 16 * c16 + x;
          sO[t * kD + lrow] =
              __float2bfloat16_rn(p.scale * (gm[t] * __uint_as_float(r1[x]) + __uint_as_float(r2[x])));
        }
      }
      return okw;
    };
    auto o_rows = [&](int cj) {
      const int cc0 = cj * kC;
      const int nn = (n_tok - cc0) < kC ? (n_tok - cc0) : kC;
      for (int idx = tid; idx < kC * 16; idx += kThreads) {
        const int t = idx >> 4, ch = idx & 15;
        if (t < nn)
          *reinterpret_cast<uint4*>(og + ((int64_t)(t0 + cc0 + t) * H + h) * kD + ch * 8) =
              *reinterpret_cast<const uint4*>(sO + t * kD + ch * 8);
      }
    };

    if (n_chunks > 0) stage(0);
#pragma unroll 1
    for (int ci = 0; ci < n_chunks; ++ci) {
      const uint32_t bq = sb + (ci & 1) * kBufBytes + kOffQK;  // Q rows
      const uint32_t bk = bq + kC * 128;                        // K rows (same panels)
      const uint32_t bv = sb + (ci & 1) * kBufBytes + kOffV;
      const uint32_t btw = sb + (ci & 1) * kBufBytes + kOffTw;
      // the next chunk into the other buffer (chunk ci - 1 is done with it), then chunk ci
      if (ci + 1 < n_chunks) stage(ci + 1);
      const bool okl = mbar_wait(&bars[3 + (ci & 1)], (lpar >> (ci & 1)) & 1u);
      lpar ^= 1u << (ci & 1);
      pending &= ~(1u << (ci & 1));
      // rows past the end of the sequence: zero (they hold the next tokens of the array)
      const int nrow = (n_tok - ci * kC) < kC ? (n_tok - ci * kC) : kC;
      if (nrow < kC && worker) {
        unsigned char* buf = smem + (ci & 1) * kBufBytes;
        for (int idx = tid; idx < (kC - nrow) * 16; idx += kWorkers) {
          const int r = nrow + (idx >> 4), ch = idx & 15;
          *reinterpret_cast<uint4*>(buf + kOffQK + umma::panel_piece(128, r, ch)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(buf + kOffQK + umma::panel_piece(128, r + kC, ch)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(buf + kOffV + umma::panel_piece(kC, r, ch)) = make_uint4(0, 0, 0, 0);
        }
      }
      // ---- this chunk's gate quantities, from the workspace tile; gamma_t also kept for the
      //      output epilogue, which runs during the next chunk
      const float* gbk = reinterpret_cast<const float*>(smem + (ci & 1) * kBufBytes + kOffGB);
      if (tid < kC) reinterpret_cast<float*>(smem + kOffGo)[(ci & 1) * kC + tid] = gbk[tid];
      const float* sGu = gbk + kC;       // gamma_C / gamma_t
      const float* sFa = gbk + 2 * kC;   // gamma_t / e^m
      const float* sFb = gbk + 3 * kC;   // e^m / gamma_t
      const float* sLg = gbk + 4 * kC;   // log |gamma_t|
      const float* sSg = gbk + 5 * kC;   // sign gamma_t
      umma::fence_smem();  // zeroed rows -> tensor cores
      if (__syncthreads_or(!okl)) {
        abort = true;
        break;
      }
      const bool fact = gbk[6 * kC] != 0.0f;
      const float gC = gbk[kC - 1];  // gamma_C (padded tokens have gate 1: the last real token's)

      // ---- MMAs, group 1 (descriptors: one per operand matrix, stepped by constant byte
      //      offsets).  P = [Q; K] K^T, W^T = K^T Tw^T and U^T = V^T Tu^T need no state:
      //      they go first and run beside the S pass; P and W^T are all the first epilogue
      //      needs, so their commit comes before U~ (group 2's commit covers the rest: the
      //      tensor core keeps issue order).  O1^T = S0^T Q^T follows the S pass.
      const uint64_t dQK = umma::sdesc(bq, 16, 1024);     // [Q; K] rows, K-major
      const uint64_t dKm = umma::sdesc(bk, 16384, 1024);  // K as an MN-major operand
      const uint64_t dS = umma::sdesc(sb + kOffS, 16, 1024);
      if (tid == kWorkers) {
        umma::fence_after();
        const uint64_t dVm = umma::sdesc(bv, 8192, 1024);
        const uint64_t dTw = umma::sdesc(btw, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = d_k
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma::mma(tmem + kColP, umma::sdesc_add(dQK, ko), umma::sdesc_add(dQK, 8192 + ko), kIdKK64, kk);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = tokens
          umma::mma(tmem + kColW, umma::sdesc_add(dKm, kk * 2048), umma::sdesc_add(dTw, kk * 32), kIdMK64, kk);
        umma::commit(&bars[0]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = tokens
          umma::mma(tmem + kColU, umma::sdesc_add(dVm, kk * 2048), umma::sdesc_add(dTw, 8192 + kk * 32), kIdMK64,
                    kk);
      }

      // ---- S pass: BF16 copy of S0^T for this chunk's products, then S^T *= gamma_C
#pragma unroll 1
      for (int c16 = 0; c16 < (worker ? 4 : 0); ++c16) {
        uint32_t r[16];
        umma::ld16(tq + kColS + 64 * hf + 16 * c16, r);
        umma::wait_ld();
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
          *reinterpret_cast<uint4*>(smem + kOffS + umma::panel_piece(128, lrow, 8 * hf + 2 * c16 + pc)) =
              pack8(r + 8 * pc);
        if (kGate) {
#pragma unroll
          for (int x = 0; x < 16; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * gC);
          umma::st16(tq + kColS + 64 * hf + 16 * c16, r);
        }
      }
      if (kGate && worker) umma::wait_st();
      const bool okt = ci > 0 ? o_tile(ci - 1) : true;  // beside group 1
      umma::fence_smem();
      umma::fence_before();
      if (__syncthreads_or(!okt)) {
        abort = true;
        break;
      }
      if (tid == kWorkers) {
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = d_k
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma::mma(tmem + kColO1 + 64 * (ci & 1), umma::sdesc_add(dS, ko), umma::sdesc_add(dQK, ko), kIdKK64, kk);
        }
      }
      bool ok = mbar_wait(&bars[0], phase & 1u);
      umma::fence_after();
      // W^T rows (lane = d_k index) -> shared memory, the B operand of the U update
#pragma unroll
      for (int c16 = 0; c16 < (worker ? 2 : 0); ++c16) {
        uint32_t r[16];
        umma::ld16(tq + kColW + 32 * hf + 16 * c16, r);
        umma::wait_ld();
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
          *reinterpret_cast<uint4*>(smem + kOffW + umma::panel_piece(128, lrow, 4 * hf + 2 * c16 + pc)) =
              pack8(r + 8 * pc);
      }
      // P rows (lanes 0..63 = token t): masked by the gate ratios
      if (worker && q4 < 2) {
        const int t = lrow;
#pragma unroll
        for (int c16 = 0; c16 < 2; ++c16) {
          uint32_t r[16];
          umma::ld16(tq + kColP + 32 * hf + 16 * c16, r);
          umma::wait_ld();
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int s = 32 * hf + 16 * c16 + x;
            float v = 0.0f;
            if (s <= t)
              v = (fact ? sFa[t] * sFb[s] : sSg[t] * sSg[s] * __expf(sLg[t] - sLg[s])) * __uint_as_float(r[x]);
            r[x] = __float_as_uint(v);
          }
#pragma unroll
          for (int pc = 0; pc < 2; ++pc)
            *reinterpret_cast<uint4*>(smem + kOffP + umma::panel_piece(kC, t, 4 * hf + 2 * c16 + pc)) =
                pack8(r + 8 * pc);
        }
      }
      umma::fence_smem();
      umma::fence_before();
      if (__syncthreads_or(!ok)) {
        abort = true;
        break;
      }

      // ---- group 2: U^T -= S0^T W^T
      if (tid == kWorkers) {
        umma::fence_after();
        const uint64_t dWm = umma::sdesc(sb + kOffW, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = d_k
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma::mma(tmem + kColU, umma::sdesc_add(dS, ko), umma::sdesc_add(dWm, kk * 2048), kIdKM64n, 1);
        }
        umma::commit(&bars[1]);
      }
      if (ci > 0) o_rows(ci - 1);  // beside group 2
      __syncthreads();              // the U space is rewritten below
      ok = mbar_wait(&bars[1], phase & 1u);
      umma::fence_after();
      // U^T rows (lane = d_v index) -> U and Us = U (gamma_C / gamma_t) per token column
#pragma unroll
      for (int c16 = 0; c16 < (worker ? 2 : 0); ++c16) {
        uint32_t r[16];
        umma::ld16(tq + kColU + 32 * hf + 16 * c16, r);
        umma::wait_ld();
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
          *reinterpret_cast<uint4*>(smem + kOffU + umma::panel_piece(128, lrow, 4 * hf + 2 * c16 + pc)) =
              pack8(r + 8 * pc);
#pragma unroll
        for (int x = 0; x < 16; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * sGu[32 * hf + 16 * c16 + x]);
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
          *reinterpret_cast<uint4*>(smem + kOffUs + umma::panel_piece(128, lrow, 4 * hf + 2 * c16 + pc)) =
              pack8(r + 8 * pc);
      }
      umma::fence_smem();
      umma::fence_before();
      if (__syncthreads_or(!ok)) {
        abort = true;
        break;
      }

      // ---- group 3: O2^T = U^T P^T ;  S^T += Us^T K
      if (tid == kWorkers) {
        umma::fence_after();
        const uint64_t dP = umma::sdesc(sb + kOffP, 16, 1024);
        const uint64_t dU = umma::sdesc(sb + kOffU, 16, 1024);
        const uint64_t dUs = umma::sdesc(sb + kOffUs, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = tokens
          umma::mma(tmem + kColS, umma::sdesc_add(dUs, kk * 32), umma::sdesc_add(dKm, kk * 2048), kIdKM128, 1);
        umma::commit(&bars[2]);  // the state: the next chunk's S pass waits for this
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = tokens
          umma::mma(tmem + kColO2, umma::sdesc_add(dU, kk * 32), umma::sdesc_add(dP, kk * 32), kIdKK64, kk);
        umma::commit(&bars[5]);  // O2: the output epilogue, one chunk later, waits for this
      }
      ok = mbar_wait(&bars[2], phase & 1u);
      umma::fence_after();
      umma::fence_smem();  // this chunk's reads of its staging buffer precede the copies into it
      umma::fence_before();
      if (__syncthreads_or(!ok)) {
        abort = true;
        break;
      }
      ++phase;
    }
    if (abort) break;
    if (n_chunks > 0) {
      const bool okt = o_tile(n_chunks - 1);
      if (__syncthreads_or(!okt)) {
        abort = true;
        break;
      }
      o_rows(n_chunks - 1);
    }

    // ---- final state: S[i][j] = S^T[j][i], lane j, columns i
    const int64_t dbase = ((int64_t)ws * H + h) * (kD * kD);
#pragma unroll 1
    for (int c16 = 0; c16 < (worker ? 4 : 0); ++c16) {
      uint32_t r[16];
      umma::ld16(tq + kColS + 64 * hf + 16 * c16, r);
      umma::wait_ld();
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int64_t e = dbase + (int64_t)(64 * hf + 16 * c16 + x) * kD + lrow;
        if (p.dst_dtype == LA_F32)
          static_cast<float*>(p.dst)[e] = __uint_as_float(r[x]);
        else
          static_cast<__nv_bfloat16*>(p.dst)[e] = __float2bfloat16_rn(__uint_as_float(r[x]));
      }
    }
    umma::fence_smem();  // this unit's reads of the staging buffers precede the next unit's copies
    umma::fence_before();
    __syncthreads();
  }

  // copies still in flight (only after a wait gave up): let them land, within the limit;
  // and every MMA issued completes before the tensor memory is released
  if (tid == kWorkers) {
    for (int b = 0; b < 2; ++b)
      if (pending & (1u << b)) mbar_wait(&bars[3 + b], (lpar >> b) & 1u);
    umma::commit(&bars[6]);
    mbar_wait(&bars[6], 0);
  }
  if (abort && tid == 0) report(p.err, LA_DEVERR_TIMEOUT);
  umma::fence_before();
  __syncthreads();
  if (warp == 0) umma::dealloc(tmem, kTmemCols);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline EncodeTiledFn encode_tiled_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// [tokens][heads][128] BF16 rows as the 3-D array {128, heads, tokens}: 64 x 64 panels
// with the 128-byte swizzle; reads past the last token return zero.
inline bool encode_rows_map(CUtensorMap* m, const void* base, int heads, int64_t tokens) {
  const EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)(tokens > 0 ? tokens : 1)};
  const cuuint64_t strides[2] = {256, (cuuint64_t)heads * 256};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t elem[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int RULE>
cudaError_t launch_chunk_tc(const ScanParams& p, cudaStream_t stream) {
  const void* fn = reinterpret_cast<const void*>(&chunk_tc_kernel<RULE>);
  const int per_sm = prepare_kernel(fn, chunk_tc::kThreads, chunk_tc::kSmem);
  // one CTA per SM: the kernel holds all of the SM's tensor memory
  if (per_sm != 1) return cudaErrorInvalidConfiguration;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));  // no tokens: nothing is staged, the maps are never read
  if (p.total_tokens > 0 &&
      (!encode_rows_map(&maps.q, p.q, p.n_qk_heads, p.total_tokens) ||
       !encode_rows_map(&maps.k, p.k, p.n_qk_heads, p.total_tokens) ||
       !encode_rows_map(&maps.v, p.v, p.n_v_heads, p.total_tokens)))
    return cudaErrorInvalidValue;
  const int64_t units = (int64_t)p.n_seqs * p.n_v_heads;
  const int64_t cap = device_sm_count();
  const int grid = (int)(units < cap ? units : cap);
  chunk_tc_kernel<RULE><<<grid, chunk_tc::kThreads, chunk_tc::kSmem, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace la
