// la_chunk_fused.cuh -- the chunked (WY / UT) prefill in one launch on the fifth-generation
// tensor cores, with every intra-chunk quantity kept on chip.
//
// Algebra ("Seven Architectures Replacing KV Cache With Bounded Mutable State": the "Kimi
// Linear" section's chunkwise-parallel kernel, the "Gated DeltaNet-2" section's chunkwise
// WY algorithm).  Per (sequence, head) and chunk of C = 64 tokens, with S0 the state at the
// chunk start, gamma_t the product of the chunk's decays up to token t and b_t the write
// strength of the rule:
//
//   L  = strictly-lower( b_t (gamma_t / gamma_s) k_t . k_s ),   T = (I + L)^-1
//   W  = T diag(b gamma) K,    U~ = T diag(b) V,    U = U~ - W S0      (delta rules; else U = V)
//   O  = scale ( Q~ S0 + P U ),   Q~ = diag(gamma) Q,   P = (Q K^T) (.) M,  M_ts = gamma_t / gamma_s (s <= t)
//   S  = gamma_C S0 + K^T Us,     Us = diag(gamma_C / gamma) U     (rules without inverse: K~^T V,
//                                                                    K~ = diag(gamma_C / gamma) K)
//
// which unrolls the token recurrence u_t = b (v_t - c S_{t-1}^T k_t), S_t = a S_{t-1} + k_t u_t^T
// exactly.  Every product is an M = 128 tcgen05 MMA with BF16 operands and an FP32
// accumulator in tensor memory; the transposed forms (U^T, O^T, S^T: one d_v index per
// tensor-memory lane) let the state, its BF16 copy S0^T and the BF16 copies of U^T and Us^T
// feed the next products straight from tensor memory as the A operand.
//
// One CTA of 14 warps per SM, each role a pipeline stage joined by mbarriers:
//   warp 0       loads: Q, K, V of a chunk by TMA tensor maps into one of three stages;
//                its lanes read the chunk's gates and write the stage's gate block
//                (prefix products of the decays, their factored ratios, b_t)
//   warp 1       lane 0 issues every MMA (and owns the tensor-memory allocation)
//   warps 2-5    intra-chunk work, ahead of the state: P and L from [Q; K] K^T,
//                T = (I + L)^-1 (16 x 16 diagonal blocks by FP32 substitution, off-diagonal
//                blocks by TF32 MMA), then Tw = T diag(b gamma), Tu = T diag(b) in one pass;
//                for the rules without inverse Q~ and K~ in place
//   warps 6-9    the state: S0^T -> BF16 copy and S^T *= gamma_C per chunk, U^T -> BF16
//                U^T and Us^T, initial and final states
//   warps 10-13  W^T -> shared memory and Q~ in place (delta rules), outputs (staged in
//                shared memory, written as 16-byte pieces of whole rows)
// The per-iteration code of every role is kept compact (rolled loops): the four roles share
// each SM sub-partition's instruction cache, and unrolled epilogues thrashed it.  A group
// waits on an mbarrier through one polling thread; the others sleep on the group's named
// barrier.
// Per chunk j the issuer runs: W_j and U~_j (after the intra-chunk work of chunk j),
// U_j -= S0^T W^T, O_j = S0^T Q~^T, then S^T += Us^T K and O_j += U^T P^T, then [Q; K] K^T of
// chunk j + 2.  Every wait has a time limit and a CTA-wide abort flag: a wait that gives up
// stops every role, the issuer drains its MMAs, the loader its copies, and the kernel
// reports LA_DEVERR_TIMEOUT.  Units (sequence, head) are dealt to the CTAs in a fixed
// boustrophedon order over seq_order (longest first balances the load).
#pragma once

#include <cstdint>
#include <cstring>

#include "la_chunk.cuh"
#include "la_chunk_tc.cuh"
#include "la_umma.cuh"

namespace la {
namespace fused {

constexpr int kC = 64;   // tokens per chunk
constexpr int kD = 128;  // d_k = d_v
constexpr int kStages = 3;

// warp roles
constexpr int kWarpLoad = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpPrep = 2;   // warps 2..5
constexpr int kWarpState = 6;  // warps 6..9
constexpr int kWarpOut = 10;   // warps 10..13
constexpr int kWarpConv = 14;  // warps 14, 15 (with the convolution)
constexpr int kThreads = 14 * 32;
constexpr int kThreadsConv = 16 * 32;
// named barriers of the warp groups (0 is __syncthreads)
constexpr uint32_t kNbPrep = 1, kNbState = 2, kNbOut = 3, kNbConv = 4;

// shared memory (bytes from a 1024-byte aligned base); BF16 operands in 64-column panels
constexpr int kStageBytes = 49152;
constexpr int kOffQK = 0;      // in a stage: two panels of 128 rows, Q rows 0..63, K rows 64..127
constexpr int kOffV = 32768;   //             two panels of 64 rows
constexpr int kOffWt = kStages * kStageBytes;  // W^T [128 d_k][64 t]; the outputs' staging tile
constexpr int kOffP = kOffWt + 16384;          // P [2][64 t][64 s] (chunk parity)
constexpr int kOffTw = kOffP + 2 * 8192;       // Tw [64 t][64 s]
constexpr int kOffTu = kOffTw + 8192;          // Tu [64 t][64 s]
constexpr int kLs = kC + 4;                    // padded row stride of L / T (fp32)
constexpr int kOffL = kOffTu + 8192;           // L, then T in place [64][68] fp32
constexpr int kXs = chunk::kXs;
constexpr int kOffX = kOffL + kC * kLs * 4;    // [3][16][24] fp32, scratch of the block recursion
// gate block of a stage (written by the loader): [0, 64) gamma_t, [64, 128) gamma_C / gamma_t,
// [128, 192) A_t = gamma_t / e^m, [192, 256) B_t = e^m / gamma_t, [256, 320) log |gamma_t|,
// [320, 384) sign gamma_t, [384, 448) b_t, [448] 1 when gamma_t / gamma_s = A_t B_s may be used
constexpr int kGB = 7 * kC + 4;                         // floats per gate block
constexpr int kOffGB = kOffX + 3 * 16 * kXs * 4;        // [kStages][kGB] fp32
constexpr int kOffBar = kOffGB + kStages * kGB * 4;
enum Bar {
  kFull = 0,        // [3] stage loaded (TMA bytes + 32 lane arrivals of the gate block)
  kEmpty = 3,       // [3] stage free (MMA commit)
  kG1Full = 6,      // [Q; K] K^T of a chunk in tensor memory (MMA commit)
  kG1Free,          // the intra-chunk group has read it
  kPrepDone,        // Tw, Tu and P ready (rules without inverse: P, Q~ and K~)
  kWFull,           // W^T and U~^T in tensor memory (MMA commit)
  kWFree,           // W^T is in shared memory
  kQt,              // Q~ ready (delta rules)
  kSPass,           // S0^T copied to BF16 and S^T scaled by gamma_C
  kUFull,           // U^T in tensor memory (MMA commit)
  kUDone,           // U^T and Us^T copied to BF16
  kSFull,           // state update done (MMA commit)
  kOFull,           // outputs of a chunk in tensor memory (MMA commit)
  kOFree,           // outputs read
  kDrain,           // every MMA issued has completed
  kConvDone,        // the convolution of a chunk's q, k, v is in its stage (with the convolution)
  kNumBars
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // [0] tensor-memory base, [1] abort
constexpr int kSmem = kOffMisc + 16 + 1024;       // + slack for the 1024-byte alignment
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kOffWt % 1024 == 0 && kOffP % 1024 == 0 && kOffTw % 1024 == 0 && kOffL % 16 == 0 &&
                  kOffGB % 16 == 0 && (kGB * 4) % 16 == 0 && kOffBar % 8 == 0,
              "alignment");

// bytes the TMA engine writes into a stage per chunk: Q, K, V (two 64 x 64 panels each)
constexpr uint32_t kTmaBytes = 6 * kC * 128;

// tensor-memory columns (FP32 accumulators unless noted; 128 lanes each)
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0;      // S^T        [d_v][d_k]     128
constexpr int kColSb = 128;   // S0^T BF16  [d_v][d_k / 2]  64 (A operand)
constexpr int kColG1 = 192;   // [Q; K] K^T [128][64]       64
constexpr int kColW = 256;    // W^T        [d_k][64]       64
constexpr int kColU = 320;    // U^T        [d_v][64]       64
constexpr int kColUb = 384;   // U^T BF16   [d_v][32]       32 (A operand)
constexpr int kColUsb = 416;  // Us^T BF16  [d_v][32]       32 (A operand)
constexpr int kColO = 448;    // O^T        [d_v][64]       64

// D (tensor memory) = A (tensor memory, BF16 packed two per column) B (shared memory)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// mbarrier phase test that lets the hardware suspend the thread (up to about `hint_ns`)
// until the phase completes, instead of returning at once
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// A pipeline wait with a time limit and the CTA's abort flag: false when it gave up (the
// flag is then set) or another role gave up first.  Called by ONE thread of a group: the
// others wait on the group's named barrier (gwait), which costs no shared-memory traffic.
__device__ __forceinline__ bool fwait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t polls = 1;; ++polls) {
    if (mbar_try_wait_hint(bar, parity, 200000u)) return true;
    if (*abort_flag) return false;
    if (polls >= kWaitMaxPolls || global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1u;
      return false;
    }
  }
}

// The same for a warp group of 128 threads: thread 0 of the group polls, every thread leaves
// with the same answer (true: the phase completed; false: abort).
__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, int tp,
                                      uint32_t nb) {
  bool ok = true;
  if (tp == 0) ok = fwait(bar, parity, abort_flag);
  return !named_bar_or(nb, 128, !ok);
}

// q8 pools (d_k = d_v = 128): row i of a head is BF16 (idx = its rank among the BF16 rows)
// or INT8 (idx = its rank among the INT8 rows), as the head's mask says
__device__ __forceinline__ bool q8_row(const uint32_t* mask, int h, int i, int& idx) {
  int below = 0;
  uint32_t word = 0u;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t m = __ldg(mask + h * 4 + w);
    if (w < (i >> 5)) below += __popc(m);
    if (w == (i >> 5)) word = m;
  }
  const int b = i & 31;
  const int pre = below + __popc(word & ((1u << b) - 1u));
  const bool hp = (word >> b) & 1u;
  idx = hp ? pre : i - pre;
  return hp;
}

// S[i][r] of a q8 tile `tl` (n8 INT8 rows) -- kept out of line, with scalar arguments, so that
// the state group's loop stays compact for the instruction cache
__device__ __noinline__ float q8_load_elem(const unsigned char* tl, int n8, const uint32_t* mask, int h, int i, int r) {
  int idx;
  if (q8_row(mask, h, i, idx))
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(tl + n8 * 128 + n8 * 16)[idx * 128 + r]);
  return __fmul_rn((float)(int)(int8_t)tl[idx * 128 + r],
                   *reinterpret_cast<const float*>(tl + n8 * 128 + (idx * 4 + (r >> 5)) * 4));
}

// S[i][r] = y into a q8 tile: the warp's 32 lanes hold row i's 32-column group r / 32, whose
// absmax sets its scale (called by whole warps, all with the same i)
__device__ __noinline__ void q8_store_elem(unsigned char* tl, int n8, const uint32_t* mask, int h, int i, int r, float y) {
  int idx;
  if (q8_row(mask, h, i, idx)) {
    reinterpret_cast<__nv_bfloat16*>(tl + n8 * 128 + n8 * 16)[idx * 128 + r] = __float2bfloat16_rn(y);
    return;
  }
  float amax = fabsf(y);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  float sc, inv;
  q8_scales(amax, sc, inv);
  tl[idx * 128 + r] = (unsigned char)q8_code(y, inv);
  if ((r & 31) == 0) *reinterpret_cast<float*>(tl + n8 * 128 + (idx * 4 + (r >> 5)) * 4) = sc;
}

// One (sequence, head) unit: its tokens, slots and whether it can be processed.
struct Unit {
  int seq, h, hq, t0, n_tok, rs, ws;
  uint32_t err;  // bits to report (also for some processed units: cu_seqlens[0] != 0)
  bool valid;
};

__device__ __forceinline__ Unit unit_info(const ScanParams& p, int64_t u) {
  Unit x;
  const int H = p.n_v_heads;
  const int64_t si = u / H;
  x.h = (int)(u % H);
  x.hq = x.h / (H / p.n_qk_heads);
  x.seq = p.seq_order ? __ldg(p.seq_order + si) : (int)si;
  x.err = 0u;
  x.valid = false;
  x.t0 = x.n_tok = x.rs = x.ws = 0;
  if (x.seq < 0 || x.seq >= p.n_seqs) {
    x.err = LA_DEVERR_CU_SEQLENS;
    return x;
  }
  const int t0 = __ldg(p.cu_seqlens + x.seq), t1 = __ldg(p.cu_seqlens + x.seq + 1);
  if (x.seq == 0 && x.h == 0 && t0 != 0) x.err |= LA_DEVERR_CU_SEQLENS;
  if (t0 < 0 || t1 < t0 || t1 > p.total_tokens) {
    x.err |= LA_DEVERR_CU_SEQLENS;
    return x;
  }
  x.rs = p.read_slot ? __ldg(p.read_slot + x.seq) : 0;
  x.ws = p.write_slot ? __ldg(p.write_slot + x.seq) : x.seq;
  const bool rs_ok = !p.read_slot || (x.rs >= 0 && x.rs < p.src_slots);
  const bool ws_ok = x.ws >= 0 && x.ws < p.dst_slots;
  if (!rs_ok || !ws_ok) {
    x.err |= (rs_ok ? 0u : LA_DEVERR_READ_SLOT) | (ws_ok ? 0u : LA_DEVERR_WRITE_SLOT);
    return x;
  }
  // q8 pools: the head's masks must mark exactly n_hp rows, or the row ranks leave the tile
  if ((p.read_slot && p.src_dtype == LA_Q8) || p.dst_dtype == LA_Q8) {
    int cs = p.src_n_hp, cd = p.dst_n_hp;
    for (int w = 0; w < 4; ++w) {
      if (p.read_slot && p.src_dtype == LA_Q8) cs -= __popc(__ldg(p.src_mask + x.h * 4 + w));
      if (p.dst_dtype == LA_Q8) cd -= __popc(__ldg(p.dst_mask + x.h * 4 + w));
    }
    if (cs != 0 || cd != 0) {
      x.err |= LA_DEVERR_Q8_MASK;
      return x;
    }
  }
  x.t0 = t0;
  x.n_tok = t1 - t0;
  x.valid = true;
  return x;
}

// the unit of round r for CTA b: boustrophedon over the grid
__device__ __forceinline__ int64_t unit_of(int64_t r, int64_t G, int64_t b) {
  return r * G + ((r & 1) ? (G - 1 - b) : b);
}

__device__ __forceinline__ uint32_t pack2(uint32_t lo, uint32_t hi) {
  return pack_bf16x2(__uint_as_float(lo), __uint_as_float(hi));
}

// rows [row0, row0 + 64) of a stage's [Q; K] panel pair scaled in place, row t by f[t] (rows
// at or past nv zeroed when zero_tail), by the 128 threads of a group (tp = 0..127):
// Q~ = diag(gamma) Q, K~ = diag(gamma_C / gamma) K
__device__ __forceinline__ void scale_rows(unsigned char* st, int row0, const float* f, int nv, bool zero_tail,
                                           int tp) {
#pragma unroll 4
  for (int i = 0; i < 8; ++i) {
    const int idx = tp + 128 * i;
    const int t = idx >> 4, ch = idx & 15;
    uint4* ptr = reinterpret_cast<uint4*>(st + umma::panel_piece(128, row0 + t, ch));
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (!zero_tail || t < nv) {
      const uint4 v = *ptr;
      const float ft = f[t];
      w = make_uint4(pack_bf16x2(bf16_lo(v.x) * ft, bf16_hi(v.x) * ft), pack_bf16x2(bf16_lo(v.y) * ft, bf16_hi(v.y) * ft),
                     pack_bf16x2(bf16_lo(v.z) * ft, bf16_hi(v.z) * ft), pack_bf16x2(bf16_lo(v.w) * ft, bf16_hi(v.w) * ft));
    }
    *ptr = w;
  }
}

}  // namespace fused

// CONV: the short causal convolution (and SiLU, q/k unit length) runs on the raw q, k, v of
// each staged chunk, in place, in a group of two more warps (14, 15) as soon as the chunk has
// landed: thread tc owns the channel pair (2 tc, 2 tc + 1) of q, k and v for a whole unit,
// with its weights and the window of its last W - 1 raw inputs in registers (read from the
// history at the read slot when the unit starts, written to the history at the write slot
// when it ends).  The issuer forms a chunk's [Q; K] K^T only once its convolution is done.
template <int RULE, bool CONV = false>
__global__ void __launch_bounds__(CONV ? fused::kThreadsConv : fused::kThreads, 1)
    chunk_fused_kernel(const ScanParams p,
                                                                         const __grid_constant__ TcMaps maps) {
  using namespace fused;
  constexpr bool kDelta = Rule<RULE>::kPredicts;
  constexpr bool kGate = Rule<RULE>::kUsesGate;
  static_assert(!Rule<RULE>::kChannelGate, "scalar gates only");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = misc + 1;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int H = p.n_v_heads;
  const int64_t units = (int64_t)p.n_seqs * H;
  const int64_t G = gridDim.x;

  if (warp == kWarpMma) umma::alloc(const_cast<uint32_t*>(misc), kTmemCols);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kFull + s], 33);
      mbar_init(&bars[kEmpty + s], 1);
    }
    for (int b = kG1Full; b < kNumBars; ++b) mbar_init(&bars[b], 1);
    misc[1] = 0u;
    mbar_init_fence();
  }
  // the strictly upper 16 x 16 blocks of Tw and Tu stay zero in every chunk
  if (kDelta && warp >= kWarpPrep && warp < kWarpState) {
    for (int idx = tid - kWarpPrep * 32; idx < kC * kC / 2; idx += 128) {
      const int r = idx >> 5, c = 2 * (idx & 31);
      if ((c >> 4) > (r >> 4)) {
        const uint32_t off = umma::panel_off(kC, r, c);
        *reinterpret_cast<uint32_t*>(smem + kOffTw + off) = 0u;
        *reinterpret_cast<uint32_t*>(smem + kOffTu + off) = 0u;
      }
    }
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
    for (int64_t r = 0; ok && r * G < units; ++r) {
      const int64_t u = unit_of(r, G, blockIdx.x);
      if (u >= units) continue;
      const Unit x = unit_info(p, u);
      if (!x.valid) continue;
      const int nch = (x.n_tok + kC - 1) / kC;
      // the query head: of the q/k head, or query q_index of the state head's group
      const int qhead = p.q_group > 1 ? x.h * p.q_group + p.q_index : x.hq;
      for (int c = 0; c < nch; ++c, ++j) {
        const int s = (int)(j % kStages);
        const int tok0 = x.t0 + c * kC;
        const int nv = min(kC, x.n_tok - c * kC);
        // the chunk's gates: tokens 2 lane and 2 lane + 1 (padded tokens: no decay, no write)
        float gi[2] = {1.0f, 1.0f}, bi[2] = {0.0f, 0.0f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 2 * lane + e;
          if (t < nv) {
            const int64_t ix = (int64_t)(tok0 + t) * H + x.h;
            gi[e] = kGate ? __ldg(p.g + ix) : 1.0f;
            bi[e] = Rule<RULE>::kUsesBeta ? __ldg(p.beta + ix) : 1.0f;
          }
        }
        if (j >= kStages && lane == 0) ok = fwait(&bars[kEmpty + s], (uint32_t)((j / kStages) + 1) & 1u, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        unsigned char* st = smem + s * kStageBytes;
        if (lane == 0) {
          uint64_t* full = &bars[kFull + s];
          mbar_arrive_expect_tx(full, kTmaBytes);
#pragma unroll
          for (int pnl = 0; pnl < 2; ++pnl) {
            umma::tma_load_3d(st + kOffQK + pnl * 16384, &maps.q, 64 * pnl, qhead, tok0, full);
            umma::tma_load_3d(st + kOffQK + pnl * 16384 + kC * 128, &maps.k, 64 * pnl, x.hq, tok0, full);
            umma::tma_load_3d(st + kOffV + pnl * 8192, &maps.v, 64 * pnl, x.h, tok0, full);
          }
        }
        // gate block: prefixes of log |a| and of the sign over the chunk, the factored
        // ratios gamma_t / gamma_s = A_t B_s around the chunk's middle (when the chunk's
        // gates are at most 1 in magnitude and span at most e^80), b_t
        float* gbk = reinterpret_cast<float*>(smem + kOffGB) + s * kGB;
        float lg[2], sg[2];
        bool big = false;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 2 * lane + e;
          float a, bc, cc;
          Rule<RULE>::coeffs(gi[e], bi[e], a, bc, cc);
          if (t >= nv) bc = 0.0f;  // padded tokens write nothing
          big |= fabsf(a) > 1.0f;
          lg[e] = __logf(fmaxf(fabsf(a), 1e-30f));
          sg[e] = a < 0.0f ? -1.0f : 1.0f;
          gbk[6 * kC + t] = bc;
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
        const float lprev = l - (lg[0] + lg[1]), sprev = sgn * sg[0] * sg[1];
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
        if (lane == 0) gbk[7 * kC] = fact ? 1.0f : 0.0f;
        mbar_arrive(&bars[kFull + s]);  // release: this lane's gate-block writes
      }
    }
    // copies still in flight (after an abort): let them land, within the limit
    if (lane == 0) {
      for (int64_t jj = (j > kStages ? j - kStages : 0); jj < j; ++jj)
        mbar_wait(&bars[kFull + (int)(jj % kStages)], (uint32_t)(jj / kStages) & 1u);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdKK64 = umma::idesc_bf16(128, 64, false, false);        // A, B K-major
      constexpr uint32_t kIdMK64 = umma::idesc_bf16(128, 64, true, false);         // A MN-major
      constexpr uint32_t kIdTM64n = umma::idesc_bf16(128, 64, false, true, true);  // A tmem, B MN, -A
      constexpr uint32_t kIdTK64 = umma::idesc_bf16(128, 64, false, false);        // A tmem, B K-major
      constexpr uint32_t kIdTM128 = umma::idesc_bf16(128, 128, false, true);       // A tmem, B MN-major
      constexpr uint32_t kIdMM128 = umma::idesc_bf16(128, 128, true, true);        // A, B MN-major
      const uint64_t dTw = umma::sdesc(sb + kOffTw, 16, 1024);
      const uint64_t dTu = umma::sdesc(sb + kOffTu, 16, 1024);
      const uint64_t dWm = umma::sdesc(sb + kOffWt, 16384, 1024);
      auto W = [&](int b, int64_t ph) { return fwait(&bars[b], (uint32_t)ph & 1u, abort_flag); };
      // [Q; K] K^T of chunk jj (its stage has landed)
      auto g1 = [&](int64_t jj) {
        const uint32_t st = sb + (uint32_t)(jj % kStages) * kStageBytes;
        const uint64_t dQK = umma::sdesc(st + kOffQK, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = d_k
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma::mma(tmem + kColG1, umma::sdesc_add(dQK, ko), umma::sdesc_add(dQK, 8192 + ko), kIdKK64, kk);
        }
        umma::commit(&bars[kG1Full]);
      };
      bool ok = true;
      if (n_total > 0 && (ok = W(kFull + 0, 0) && (!CONV || W(kConvDone, 0)))) {
        umma::fence_after();
        g1(0);
      }
      if (ok && n_total > 1 && (ok = W(kFull + 1, 0) && W(kG1Free, 0) && (!CONV || W(kConvDone, 1)))) {
        umma::fence_after();
        g1(1);
      }
      for (int64_t j = 0; ok && j < n_total; ++j) {
        const uint32_t st = sb + (uint32_t)(j % kStages) * kStageBytes;
        const uint64_t dQK = umma::sdesc(st + kOffQK, 16, 1024);            // [Q~; K] rows, K-major
        const uint64_t dKm = umma::sdesc(st + kOffQK + 8192, 16384, 1024);  // K (or K~) as MN-major
        const uint64_t dVm = umma::sdesc(st + kOffV, 8192, 1024);           // V as MN-major
        const uint64_t dP = umma::sdesc(sb + kOffP + (uint32_t)(j & 1) * 8192, 16, 1024);
        if (kDelta) {
          if (!(ok = W(kPrepDone, j))) break;
          umma::fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // W^T = K^T Tw^T (K = tokens)
            umma::mma(tmem + kColW, umma::sdesc_add(dKm, kk * 2048), umma::sdesc_add(dTw, kk * 32), kIdMK64, kk);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // U^T = V^T Tu^T
            umma::mma(tmem + kColU, umma::sdesc_add(dVm, kk * 2048), umma::sdesc_add(dTu, kk * 32), kIdMK64, kk);
          umma::commit(&bars[kWFull]);
          if (!(ok = W(kWFree, j) && W(kSPass, j))) break;
          umma::fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // U^T -= S0^T W^T (K = d_k)
            mma_ts(tmem + kColU, tmem + kColSb + 8 * kk, umma::sdesc_add(dWm, kk * 2048), kIdTM64n, 1);
          umma::commit(&bars[kUFull]);
          if (!(ok = W(kQt, j))) break;
        } else {
          if (!(ok = W(kPrepDone, j) && W(kSPass, j))) break;
        }
        if (j > 0 && !(ok = W(kOFree, j - 1))) break;
        umma::fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // O^T = S0^T Q~^T (K = d_k)
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ts(tmem + kColO, tmem + kColSb + 8 * kk, umma::sdesc_add(dQK, ko), kIdTK64, kk);
        }
        if (kDelta) {
          if (!(ok = W(kUDone, j))) break;
          umma::fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // S^T += Us^T K (K = tokens)
            mma_ts(tmem + kColS, tmem + kColUsb + 8 * kk, umma::sdesc_add(dKm, kk * 2048), kIdTM128, 1);
          umma::commit(&bars[kSFull]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // O^T += U^T P^T
            mma_ts(tmem + kColO, tmem + kColUb + 8 * kk, umma::sdesc_add(dP, kk * 32), kIdTK64, 1);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // S^T += V^T K~
            umma::mma(tmem + kColS, umma::sdesc_add(dVm, kk * 2048), umma::sdesc_add(dKm, kk * 2048), kIdMM128, 1);
          umma::commit(&bars[kSFull]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // O^T += V^T P^T
            umma::mma(tmem + kColO, umma::sdesc_add(dVm, kk * 2048), umma::sdesc_add(dP, kk * 32), kIdMK64, 1);
        }
        umma::commit(&bars[kOFull]);
        umma::commit(&bars[kEmpty + (int)(j % kStages)]);
        if (j + 2 < n_total) {
          if (!(ok = W(kFull + (int)((j + 2) % kStages), (j + 2) / kStages) && W(kG1Free, j + 1) &&
                     (!CONV || W(kConvDone, j + 2))))
            break;
          umma::fence_after();
          g1(j + 2);
        }
      }
      // every MMA issued completes before the tensor memory is released
      umma::commit(&bars[kDrain]);
      mbar_wait(&bars[kDrain], 0);
    }
  } else if (warp < kWarpState) {
    // ------------------------------------------------------------------ intra-chunk group
    const int wi = warp - kWarpPrep;      // 0..3 within the group
    const int tp = tid - kWarpPrep * 32;  // 0..127
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;         // this thread's tensor-memory lane
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
    float* sL = reinterpret_cast<float*>(smem + kOffL);
    float* sX = reinterpret_cast<float*>(smem + kOffX);
    int64_t j = 0;
    bool ok = true;
    for (int64_t ru = 0; ok && ru * G < units; ++ru) {
      const int64_t u = unit_of(ru, G, blockIdx.x);
      if (u >= units) continue;
      const Unit x = unit_info(p, u);
      if (!x.valid) continue;
      const int nch = (x.n_tok + kC - 1) / kC;
      for (int c = 0; c < nch; ++c, ++j) {
        const int s = (int)(j % kStages);
        const int nv = min(kC, x.n_tok - c * kC);
        unsigned char* st = smem + s * kStageBytes + kOffQK;
        const float* gbk = reinterpret_cast<const float*>(smem + kOffGB) + s * kGB;
        // rules without inverse: stay behind the state update of chunk j - 1 (the MMA issuer
        // then never falls two phases behind this group's completions)
        if (!kDelta && j > 0 && !(ok = gwait(&bars[kSFull], (uint32_t)(j - 1) & 1u, abort_flag, tp, kNbPrep))) break;
        // the stage (and its gate block), then [Q; K] K^T of the chunk
        if (!(ok = gwait(&bars[kFull + s], (uint32_t)(j / kStages) & 1u, abort_flag, tp, kNbPrep))) break;
        if (!(ok = gwait(&bars[kG1Full], (uint32_t)j & 1u, abort_flag, tp, kNbPrep))) break;
        const bool fact = gbk[7 * kC] != 0.0f;
        const float* sFa = gbk + 2 * kC;
        const float* sFb = gbk + 3 * kC;
        const float* sLg = gbk + 4 * kC;
        const float* sSg = gbk + 5 * kC;
        const float* sBt = gbk + 6 * kC;

        // P = (Q K^T) (.) M (lanes 0..63) and L (lanes 64..127, delta rules) from tensor memory
        umma::fence_after();
        if (r < kC || kDelta) {
          // row t of P (lanes 0..63: masked by gamma_t / gamma_s, s <= t) or of L (lanes
          // 64..127: b_t gamma_t / gamma_s k_t . k_s, s < t), 32 columns at a time
          const bool is_p = r < kC;
          const int t = is_p ? r : r - kC;
          const float bt = is_p ? 1.0f : sBt[t];
          const float fa = sFa[t] * bt, sgt = sSg[t] * bt, lgt = sLg[t];
          unsigned char* sP = smem + kOffP + (j & 1) * 8192;
#pragma unroll 1
          for (int c32 = 0; c32 < 2; ++c32) {
            uint32_t v[32];
            umma::ld16(tq + kColG1 + 32 * c32, v);
            umma::ld16(tq + kColG1 + 32 * c32 + 16, v + 16);
            float rt[32];  // the ratios b_t gamma_t / gamma_s of the 32 columns
            if (fact) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 fb = *reinterpret_cast<const float4*>(sFb + 32 * c32 + 4 * q);
                rt[4 * q] = fa * fb.x;
                rt[4 * q + 1] = fa * fb.y;
                rt[4 * q + 2] = fa * fb.z;
                rt[4 * q + 3] = fa * fb.w;
              }
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 lg4 = *reinterpret_cast<const float4*>(sLg + 32 * c32 + 4 * q);
                const float4 sg4 = *reinterpret_cast<const float4*>(sSg + 32 * c32 + 4 * q);
                rt[4 * q] = sgt * sg4.x * __expf(lgt - lg4.x);
                rt[4 * q + 1] = sgt * sg4.y * __expf(lgt - lg4.y);
                rt[4 * q + 2] = sgt * sg4.z * __expf(lgt - lg4.z);
                rt[4 * q + 3] = sgt * sg4.w * __expf(lgt - lg4.w);
              }
            }
            umma::wait_ld();
            // the masked entries: s <= t for P, s < t for L
            const int lim = is_p ? t - 32 * c32 : t - 32 * c32 - 1;
#pragma unroll
            for (int e = 0; e < 32; ++e) rt[e] = e <= lim ? rt[e] * __uint_as_float(v[e]) : 0.0f;
            if (is_p) {
#pragma unroll
              for (int pc = 0; pc < 4; ++pc)
                *reinterpret_cast<uint4*>(sP + umma::panel_piece(kC, t, 4 * c32 + pc)) =
                    make_uint4(pack_bf16x2(rt[8 * pc], rt[8 * pc + 1]), pack_bf16x2(rt[8 * pc + 2], rt[8 * pc + 3]),
                               pack_bf16x2(rt[8 * pc + 4], rt[8 * pc + 5]),
                               pack_bf16x2(rt[8 * pc + 6], rt[8 * pc + 7]));
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(sL + t * kLs + 32 * c32 + 4 * q) =
                    make_float4(rt[4 * q], rt[4 * q + 1], rt[4 * q + 2], rt[4 * q + 3]);
            }
          }
        }
        umma::fence_before();
        named_bar_sync(kNbPrep, 128);
        if (tp == 0) mbar_arrive(&bars[kG1Free]);

        if (!kDelta) {
          scale_rows(st, 0, gbk, nv, false, tp);        // Q~ = diag(gamma) Q
          scale_rows(st, kC, gbk + kC, nv, true, tp);   // K~ (its only reader left is the state update)
        } else {
          chunk::ut_inverse64(sL, sX, wi, lane, kNbPrep);
          // Tw and Tu of chunk j - 1 must have been read (W_{j-1} and U~_{j-1} complete)
          if (j > 0 && !(ok = gwait(&bars[kWFull], (uint32_t)(j - 1) & 1u, abort_flag, tp, kNbPrep))) break;
          // Tw = T diag(b gamma), Tu = T diag(b) (BF16), the ten lower 16 x 16 blocks: block i
          // of (0,0) (1,0) (1,1) (2,0) ... (3,3), thread tp -> row tp / 8, columns 2 (tp % 8) + {0, 1}
          const float* sGm = gbk;
          const int rb = tp >> 3, cp = 2 * (tp & 7);
#pragma unroll 2
          for (int i = 0; i < 10; ++i) {
            const int bi = i >= 6 ? 3 : i >= 3 ? 2 : i >= 1 ? 1 : 0;
            const int bj = i - (bi * (bi + 1)) / 2;
            const int row = 16 * bi + rb, col = 16 * bj + cp;
            const float2 tv = *reinterpret_cast<const float2*>(sL + row * kLs + col);
            const float b0 = sBt[col], b1 = sBt[col + 1];
            const uint32_t off = umma::panel_off(kC, row, col);
            *reinterpret_cast<uint32_t*>(smem + kOffTw + off) =
                pack_bf16x2(tv.x * b0 * sGm[col], tv.y * b1 * sGm[col + 1]);
            *reinterpret_cast<uint32_t*>(smem + kOffTu + off) = pack_bf16x2(tv.x * b0, tv.y * b1);
          }
        }
        umma::fence_smem();  // P, Tw, Tu (Q~, K~) -> tensor cores
        named_bar_sync(kNbPrep, 128);
        if (tp == 0) mbar_arrive(&bars[kPrepDone]);
      }
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
      // checkpoints (ckpt_every a multiple of the chunk): checkpoint k is the state after the
      // first (k + 1) ckpt_every tokens, k < n_ck, to dst slot ckpt_slots[ckpt_cu[seq] + k]
      int n_ck = 0, ck_base = 0;
      if (p.ckpt_every > 0) {
        ck_base = __ldg(p.ckpt_cu + x.seq);
        n_ck = __ldg(p.ckpt_cu + x.seq + 1) - ck_base;
        const int fit = x.n_tok / p.ckpt_every;
        if (n_ck < 0 || n_ck > fit) {
          if (tp == 0) report(p.err, LA_DEVERR_CU_SEQLENS);
          n_ck = n_ck < 0 ? 0 : fit;
        }
      }
      // the checkpoint slot of the state after the first `tok` tokens, or -1 (no checkpoint
      // there, or a bad slot, which is reported)
      auto ckpt_slot = [&](int tok) -> int {
        if (p.ckpt_every <= 0 || tok == 0 || tok % p.ckpt_every) return -1;
        const int k = tok / p.ckpt_every - 1;
        if (k >= n_ck) return -1;
        const int cs = __ldg(p.ckpt_slots + ck_base + k);
        if (cs < 0 || cs >= p.dst_slots) {
          if (tp == 0) report(p.err, LA_DEVERR_WRITE_SLOT);
          return -1;
        }
        return cs;
      };
      // S[i0 + e][r] of the initial state (zero without a read slot), e < 16
      auto load_col = [&](int i0, uint32_t* v) {
        if (p.read_slot && p.src_dtype == LA_Q8) {
          const unsigned char* tl = static_cast<const unsigned char*>(p.src) +
                                    ((int64_t)x.rs * H + x.h) * q8_tile_bytes(kD, kD, p.src_n_hp);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v[e] = __float_as_uint(q8_load_elem(tl, kD - p.src_n_hp, p.src_mask, x.h, i0 + e, r));
          return;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float sv = 0.0f;
          if (p.read_slot) {
            const int64_t el = ((int64_t)x.rs * H + x.h) * (kD * kD) + (int64_t)(i0 + e) * kD + r;
            sv = p.src_dtype == LA_F32 ? static_cast<const float*>(p.src)[el]
                                       : __bfloat162float(static_cast<const __nv_bfloat16*>(p.src)[el]);
          }
          v[e] = __float_as_uint(sv);
        }
      };
      // S[i0 + e][r] = v[e] (e < 16) into slot `slot` of the destination (in the query-group
      // direction by the launch of query 0 alone)
      auto store_col = [&](int slot, int i0, const uint32_t* v) {
        if (p.q_index != 0) return;
        if (p.dst_dtype == LA_Q8) {
          unsigned char* tl =
              static_cast<unsigned char*>(p.dst) + ((int64_t)slot * H + x.h) * q8_tile_bytes(kD, kD, p.dst_n_hp);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            q8_store_elem(tl, kD - p.dst_n_hp, p.dst_mask, x.h, i0 + e, r, __uint_as_float(v[e]));
          return;
        }
        const int64_t base = ((int64_t)slot * H + x.h) * (kD * kD);
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
        if (CONV) {  // its convolution history passes through (zero without a read slot)
          const int wm1 = p.conv_w - 1;
          const __nv_bfloat16* hs = static_cast<const __nv_bfloat16*>(p.conv_src) + ((int64_t)x.rs * H + x.h) * 384 * wm1;
          __nv_bfloat16* hd = static_cast<__nv_bfloat16*>(p.conv_dst) + ((int64_t)x.ws * H + x.h) * 384 * wm1;
          for (int idx = tp; idx < 384 * wm1; idx += 128) hd[idx] = p.read_slot ? hs[idx] : __float2bfloat16_rn(0.0f);
        }
        // empty sequence: the initial state (or zero) goes to the destination
#pragma unroll 1
        for (int c16 = 0; c16 < 8; ++c16) {
          uint32_t v[16];
          load_col(16 * c16, v);
          store_col(x.ws, 16 * c16, v);
        }
        continue;
      }
      // initial state S^T: lane = d_v index r, columns = d_k
#pragma unroll 1
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t v[16];
        load_col(16 * c16, v);
        umma::st16(tq + kColS + 16 * c16, v);
      }
      umma::wait_st();
      for (int c = 0; c < nch; ++c, ++j) {
        const int s = (int)(j % kStages);
        const float* gbk = reinterpret_cast<const float*>(smem + kOffGB) + s * kGB;
        // the previous chunk's state update and this chunk's gate block (the stage is not
        // reloaded before this chunk's last MMA, which waits for this group)
        if (tp == 0) {
          if (c > 0) ok = fwait(&bars[kSFull], (uint32_t)(j - 1) & 1u, abort_flag);
          if (ok) ok = fwait(&bars[kFull + s], (uint32_t)(j / kStages) & 1u, abort_flag);
        }
        if (named_bar_or(kNbState, 128, !ok)) {
          ok = false;
          break;
        }
        umma::fence_after();
        const float gC = gbk[kC - 1];  // gamma_C (padded tokens have gate 1: the last real token's)
        const int ckb = ckpt_slot(c * kC);  // a checkpoint at this chunk boundary
        // S pass: S0^T -> BF16 (the A operand of this chunk's products), S^T *= gamma_C
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          uint32_t a[16], b[16], w[16];
          umma::ld16(tq + kColS + 32 * c32, a);
          umma::ld16(tq + kColS + 32 * c32 + 16, b);
          umma::wait_ld();
          if (ckb >= 0) {
            store_col(ckb, 32 * c32, a);
            store_col(ckb, 32 * c32 + 16, b);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w[e] = pack2(a[2 * e], a[2 * e + 1]);
            w[8 + e] = pack2(b[2 * e], b[2 * e + 1]);
          }
          umma::st16(tq + kColSb + 16 * c32, w);
          if (kGate) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              a[e] = __float_as_uint(__uint_as_float(a[e]) * gC);
              b[e] = __float_as_uint(__uint_as_float(b[e]) * gC);
            }
            umma::st16(tq + kColS + 32 * c32, a);
            umma::st16(tq + kColS + 32 * c32 + 16, b);
          }
        }
        umma::wait_st();
        umma::fence_before();
        named_bar_sync(kNbState, 128);
        if (tp == 0) mbar_arrive(&bars[kSPass]);
        if (kDelta) {
          if (!(ok = gwait(&bars[kUFull], (uint32_t)j & 1u, abort_flag, tp, kNbState))) break;
          umma::fence_after();
          // U^T -> BF16 (the A operand of O += U^T P^T) and Us^T = U^T diag(gamma_C / gamma) (the
          // A operand of the state update)
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
            const float* gcg = gbk + kC + 32 * c32;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              w[e] = pack_bf16x2(__uint_as_float(a[2 * e]) * gcg[2 * e], __uint_as_float(a[2 * e + 1]) * gcg[2 * e + 1]);
              w[8 + e] = pack_bf16x2(__uint_as_float(b[2 * e]) * gcg[16 + 2 * e],
                                     __uint_as_float(b[2 * e + 1]) * gcg[16 + 2 * e + 1]);
            }
            umma::st16(tq + kColUsb + 16 * c32, w);
          }
          umma::wait_st();
          umma::fence_before();
          named_bar_sync(kNbState, 128);
          if (tp == 0) mbar_arrive(&bars[kUDone]);
        }
      }
      if (!ok) break;
      // final state S[i][r] = S^T[r][i] (and the last checkpoint when it falls on the end)
      if (!(ok = gwait(&bars[kSFull], (uint32_t)(j - 1) & 1u, abort_flag, tp, kNbState))) break;
      umma::fence_after();
      const int ckf = ckpt_slot(x.n_tok);
#pragma unroll 1
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t v[16];
        umma::ld16(tq + kColS + 16 * c16, v);
        umma::wait_ld();
        store_col(x.ws, 16 * c16, v);
        if (ckf >= 0) store_col(ckf, 16 * c16, v);
      }
      umma::fence_before();
    }
  } else if (warp < kWarpConv) {
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
        const int s = (int)(j % kStages);
        if (kDelta) {
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
          // Q~ = diag(gamma) Q in place: [Q; K] K^T, the last reader of Q, completed before W
          // (the gate block of the stage landed with it)
          if (!(ok = gwait(&bars[kFull + s], (uint32_t)(j / kStages) & 1u, abort_flag, tp, kNbOut))) break;
          scale_rows(smem + s * kStageBytes + kOffQK, 0, reinterpret_cast<const float*>(smem + kOffGB) + s * kGB,
                     kC, false, tp);
          umma::fence_smem();
          named_bar_sync(kNbOut, 128);
          if (tp == 0) mbar_arrive(&bars[kQt]);
        }
        // outputs o_t[r] = scale O^T[r][t] for the chunk's tokens: staged as a row-major
        // [64][128] BF16 tile in the W^T buffer (free: U_j, its reader, has completed), then
        // written as 16-byte pieces of whole 256-byte rows
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
              *reinterpret_cast<uint4*>(og + ((int64_t)(tok0 + t) * H * p.q_group + x.h * p.q_group + p.q_index) * kD + ch * 8) =
                  *reinterpret_cast<const uint4*>(so + t * kD + ch * 8);
          }
        }
        named_bar_sync(kNbOut, 128);  // the staging tile is read before the next W^T lands there
      }
    }
  } else if (CONV) {
    // ------------------------------------------------------------------ convolution group
    const int tc = tid - kWarpConv * 32;  // channel pair (2 tc, 2 tc + 1) of q, k and v
    const int wid = p.conv_w;
    const uint32_t piece = (uint32_t)(((2 * tc) & 63) >> 3);
    const uint32_t pair_off[3] = {kOffQK + umma::panel_off(128, 0, 2 * tc), kOffQK + umma::panel_off(128, kC, 2 * tc),
                                  kOffV + umma::panel_off(kC, 0, 2 * tc)};
    // four taps over the window of the last three raw inputs and the current one (a narrower
    // convolution's weights sit in the last taps, the others are zero)
    float w[3][2][4], win[3][2][3];
    int64_t jj = 0;
    bool ok = true;
    for (int64_t ru = 0; ok && ru * G < units; ++ru) {
      const int64_t u = unit_of(ru, G, blockIdx.x);
      if (u >= units) continue;
      const Unit x = unit_info(p, u);
      if (!x.valid || x.n_tok == 0) continue;  // an empty sequence's history: the state group
      const int nch = (x.n_tok + kC - 1) / kC;
      const __nv_bfloat16* hs =
          static_cast<const __nv_bfloat16*>(p.conv_src) + ((int64_t)x.rs * H + x.h) * 384 * (wid - 1);
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        const float* wsrc = (m == 0 ? p.conv_wq : m == 1 ? p.conv_wk : p.conv_wv) +
                            ((int64_t)(m == 2 ? x.h : x.hq) * kD + 2 * tc) * wid;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
          for (int tap = 0; tap < 4; ++tap) {
            const int src = tap - (4 - wid);  // tap multiplies x_{t-3+tap}
            w[m][e][tap] = src >= 0 ? __ldg(wsrc + e * wid + src) : 0.0f;
          }
#pragma unroll
          for (int sl = 0; sl < 3; ++sl) {
            const int src = sl - (4 - wid);  // slot sl holds x_{t-3+sl}: history entry src
            win[m][e][sl] =
                (src >= 0 && p.read_slot) ? __bfloat162float(hs[(m * kD + 2 * tc + e) * (wid - 1) + src]) : 0.0f;
          }
        }
      }
      for (int c = 0; c < nch; ++c, ++jj) {
        const int s = (int)(jj % kStages);
        bool okc = true;
        if (tc == 0) okc = fwait(&bars[kFull + s], (uint32_t)(jj / kStages) & 1u, abort_flag);
        if (named_bar_or(kNbConv, 64, !okc)) {
          ok = false;
          break;
        }
        unsigned char* st = smem + s * kStageBytes;
        const int nv = min(kC, x.n_tok - c * kC);
        // blocks of 8 tokens: the row swizzle of a panel repeats every 8 rows, so the addresses
        // within a block are constant offsets; tokens at or past nv are left as they are
#pragma unroll 1
        for (int t0 = 0; t0 < nv; t0 += 8) {
          const int nr = min(8, nv - t0);  // real tokens of the block
#pragma unroll
          for (int m = 0; m < 3; ++m) {
            const uint32_t base = pair_off[m] + t0 * 128 - (piece << 4);
            uint32_t xr[8];
#pragma unroll
            for (int v8 = 0; v8 < 8; ++v8) xr[v8] = *reinterpret_cast<const uint32_t*>(st + base + v8 * 128 + ((piece ^ v8) << 4));
            float y[2][8];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              // the inputs x_{t0-3} .. x_{t0+7}: the window, then the block's 8 rows
              float xs[11];
#pragma unroll
              for (int i = 0; i < 3; ++i) xs[i] = win[m][e][i];
#pragma unroll
              for (int v8 = 0; v8 < 8; ++v8) xs[3 + v8] = e ? bf16_hi(xr[v8]) : bf16_lo(xr[v8]);
#pragma unroll
              for (int v8 = 0; v8 < 8; ++v8)
                y[e][v8] = fmaf(w[m][e][3], xs[v8 + 3],
                                fmaf(w[m][e][2], xs[v8 + 2], fmaf(w[m][e][1], xs[v8 + 1], w[m][e][0] * xs[v8])));
              // the window after the block's real tokens: the last three of x_{t0-3} .. x_{t0+nr-1}
              if (nr == 8) {
#pragma unroll
                for (int i = 0; i < 3; ++i) win[m][e][i] = xs[8 + i];
              } else {
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                  float nw = xs[i];
#pragma unroll
                  for (int k = 1; k < 8; ++k)
                    if (nr == k) nw = xs[k + i];
                  win[m][e][i] = nw;
                }
              }
            }
            if (p.conv_act) {
#pragma unroll
              for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int v8 = 0; v8 < 8; ++v8) y[e][v8] = __fdividef(y[e][v8], 1.0f + __expf(-y[e][v8]));
            }
#pragma unroll
            for (int v8 = 0; v8 < 8; ++v8)
              if (v8 < nr)
                *reinterpret_cast<uint32_t*>(st + base + v8 * 128 + ((piece ^ v8) << 4)) = pack_bf16x2(y[0][v8], y[1][v8]);
          }
        }
        named_bar_sync(kNbConv, 64);  // every channel of the chunk is convolved
        if (p.conv_l2norm) {
          // q_t (rows 0..63) and k_t (rows 64..127) to unit length: thread tc takes rows tc, 64 + tc
#pragma unroll 1
          for (int rr = tc; rr < 128; rr += 64) {
            if ((rr & (kC - 1)) >= nv) continue;
            float ss = 0.0f;
#pragma unroll 4
            for (int ch = 0; ch < 16; ++ch) {
              const uint4 q4 = *reinterpret_cast<const uint4*>(st + kOffQK + umma::panel_piece(128, rr, ch));
              const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
              for (int e2 = 0; e2 < 4; ++e2)
                ss = fmaf(bf16_lo(qw[e2]), bf16_lo(qw[e2]), fmaf(bf16_hi(qw[e2]), bf16_hi(qw[e2]), ss));
            }
            const float rs = rsqrtf(ss + 1e-6f);
#pragma unroll 4
            for (int ch = 0; ch < 16; ++ch) {
              uint4* ptr = reinterpret_cast<uint4*>(st + kOffQK + umma::panel_piece(128, rr, ch));
              const uint4 q4 = *ptr;
              *ptr = make_uint4(pack_bf16x2(bf16_lo(q4.x) * rs, bf16_hi(q4.x) * rs),
                                pack_bf16x2(bf16_lo(q4.y) * rs, bf16_hi(q4.y) * rs),
                                pack_bf16x2(bf16_lo(q4.z) * rs, bf16_hi(q4.z) * rs),
                                pack_bf16x2(bf16_lo(q4.w) * rs, bf16_hi(q4.w) * rs));
            }
          }
          named_bar_sync(kNbConv, 64);
        }
        umma::fence_smem();  // the convolved rows -> tensor cores
        named_bar_sync(kNbConv, 64);
        // announced once the issuer has taken the previous chunk's convolution (its [Q; K] K^T
        // completed), so that the barrier's phases never run two ahead of the issuer
        if (tc == 0) {
          if (jj > 0) okc = fwait(&bars[kG1Full], (uint32_t)(jj - 1) & 1u, abort_flag);
          if (okc) mbar_arrive(&bars[kConvDone]);
        }
        if (named_bar_or(kNbConv, 64, !okc)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      // the window after the unit's last token: its history at the write slot
      __nv_bfloat16* hd = static_cast<__nv_bfloat16*>(p.conv_dst) + ((int64_t)x.ws * H + x.h) * 384 * (wid - 1);
#pragma unroll
      for (int m = 0; m < 3; ++m)
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int sl = 0; sl < 3; ++sl) {
            const int dst = sl - (4 - wid);
            if (dst >= 0) hd[(m * kD + 2 * tc + e) * (wid - 1) + dst] = __float2bfloat16_rn(win[m][e][sl]);
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

template <int RULE, bool CONV = false>
cudaError_t launch_chunk_fused(const ScanParams& p, cudaStream_t stream) {
  const void* fn = reinterpret_cast<const void*>(&chunk_fused_kernel<RULE, CONV>);
  constexpr int threads = CONV ? fused::kThreadsConv : fused::kThreads;
  const int per_sm = prepare_kernel(fn, threads, fused::kSmem);
  // one CTA per SM: the kernel holds all of the SM's tensor memory
  if (per_sm != 1) return cudaErrorInvalidConfiguration;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));  // no tokens: nothing is staged, the maps are never read
  if (p.total_tokens > 0 &&
      (!encode_rows_map(&maps.q, p.q, p.n_qk_heads * p.q_group, p.total_tokens) ||
       !encode_rows_map(&maps.k, p.k, p.n_qk_heads, p.total_tokens) ||
       !encode_rows_map(&maps.v, p.v, p.n_v_heads, p.total_tokens)))
    return cudaErrorInvalidValue;
  const int64_t units = (int64_t)p.n_seqs * p.n_v_heads;
  const int64_t cap = device_sm_count();
  const int grid = (int)(units < cap ? units : cap);
  if (grid <= 0) return cudaSuccess;
  chunk_fused_kernel<RULE, CONV><<<grid, threads, fused::kSmem, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace la
