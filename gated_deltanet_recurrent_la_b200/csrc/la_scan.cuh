// la_scan.cuh -- token-serial scan (prefill) over packed variable-length sequences.
//
// Same recurrence as the decode step (the "Gated DeltaNet" glossary page, Technical
// definition, under the ONNX LinearAttention update rules of "Seven Architectures
// Replacing KV Cache With Bounded Mutable State"), applied token after token with the
// state held on chip in FP32 for the whole sequence: it is read once at the start and
// stored once at the end (BF16 storage, FP32 compute, as on the "Recurrent state"
// glossary page).  The pages give no prefill algorithm beyond "prefill" speed-ups; this
// is the plain sequential form, bound by FP32 issue rather than by memory.
//
// Work unit: one (sequence, state head).  Each column of S evolves on its own given
// the token's k, q, gate and beta, so the unit's d_v columns are spread over warps and
// lanes with no exchange between columns:
//   * a CTA of d_v / (8 kC) warps owns one unit; lane = 4 cg + rg owns kC columns
//     (column group cg) and the rows [rg R, rg R + R), R = d_k / 4, in FP32 registers
//     (kC = 4: 128 values per lane for 128 x 128);
//   * the state is kept as S = gam * St with a running scalar gam (the product of the
//     gates since the last fold), so the update costs one FMA per element:
//     St <- St + k (u / gam)^T.  When gam leaves [2^-40, 2^40] (or reaches 0) it is
//     folded into St; it is folded once more before the final store;
//   * per token, one fused pass over the lane's elements applies the previous token's
//     update and accumulates St^T k and St^T q for the current token (the readout
//     rearrangement of the "Gated DeltaNet" page makes S^T q the old state's product):
//     three FMAs per element, the two sums kept as even / odd row partials for more
//     independent chains; two xor-shuffles finish the d_k sums across the 4 lanes;
//   * q, k (converted to FP32 in a bank-conflict-free padded layout), v, g, beta of 16
//     upcoming tokens are staged in shared memory with cp.async double buffering;
//   * optional checkpoints: every ckpt_every tokens the pending update is applied at
//     once and the state is stored to a checkpoint slot (prefix caching at KV-block
//     boundaries, "Gated DeltaNet" glossary, Why it matters);
//   * units are dealt to persistent CTAs in the order given by seq_order (longest
//     first balances best) in a boustrophedon pattern;
//   * kda (the channel-wise gate of the "Kimi Linear" section of "Seven Architectures
//     ..."): each row has its own decay, so the scalar running gate does not apply; the
//     pending update becomes x <- alpha_i x + k_i u_j (one FMUL more per element), and
//     the token's decays are folded into the staged keys of the two sums,
//     (alpha . k) and (alpha . q).  Its staging chunk is 8 tokens (four FP32 rows per
//     token instead of two);
//   * query-group direction (QGRP; the ONNX operator's query heads sharing a KV head and its
//     state): each token carries q_group queries for the unit's state head; the first is
//     read in the fused pass, each other one costs one more pass over the registers.  Its
//     staging chunk is 4 tokens.
#pragma once

#include <cstdint>

#include "la_device.cuh"
#include "la_internal.h"

#ifndef LA_SCAN_COLS
#define LA_SCAN_COLS 4
#endif
// resident units (CTAs) per SM that the scan's register budget is held to: three for the
// plain scan (168 registers, no spills: twelve warps per SM hide more of the FMA and
// shuffle latencies), two with checkpoints (whose bookkeeping would spill at three)
#ifndef LA_SCAN_MIN_BLOCKS
#define LA_SCAN_MIN_BLOCKS 3
#endif
#ifndef LA_SCAN_MIN_BLOCKS_CKPT
#define LA_SCAN_MIN_BLOCKS_CKPT 2
#endif
#ifndef LA_SCAN_MIN_BLOCKS_CONV
#define LA_SCAN_MIN_BLOCKS_CONV 2
#endif

namespace la {

template <int DK, int DV, typename IT, bool CHG = false, int QMAX = 1, bool CONV = false>
struct ScanCfg {
  static constexpr int kLG = 4;                        // lanes sharing a column group (split d_k)
  static constexpr int kC = LA_SCAN_COLS;              // columns per lane
  static constexpr int kWarpCols = (32 / kLG) * kC;    // columns per warp
  static constexpr int kR = DK / kLG;                  // rows per lane
  static constexpr int kWarps = DV >= kWarpCols ? DV / kWarpCols : 1;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTC = QMAX > 1 ? 4 : (CHG ? 8 : 16);  // tokens per staged chunk
  static constexpr int kIB = sizeof(IT);
  static constexpr int kRowStride = kR + 4;            // padded row-block stride (floats)
  static constexpr int kKP = kLG * kRowStride;         // padded FP32 key / query length
  static constexpr int kQKVecs = DK * kIB / 16;        // 16-byte pieces per q or k row
  static constexpr int kVVecs = DV * kIB / 16;
  // raw (io dtype) staging, double buffered
  static constexpr int kRawQ = 0;                      // [kTC][QMAX][DK]
  static constexpr int kRawK = kRawQ + kTC * QMAX * DK * kIB;
  static constexpr int kRawV = kRawK + kTC * DK * kIB;
  static constexpr int kRawG = kRawV + kTC * DV * kIB;
  static constexpr int kRawB = kRawG + kTC * 4;
  static constexpr int kRawA = kRawB + kTC * 4;        // kda: FP32 decays [kTC][DK]
  static constexpr int kRawBytes = kRawA + (CHG ? kTC * DK * 4 : 0);
  // converted FP32 keys / queries and k.q, double buffered.  kda adds the decays and the
  // decayed key; its "query" row is the decayed query.
  static constexpr int kCvtK = 0;
  static constexpr int kCvtQ = kCvtK + kTC * kKP * 4;         // [kTC][QMAX][kKP]
  static constexpr int kCvtKQ = kCvtQ + kTC * QMAX * kKP * 4;  // [kTC][QMAX]
  static constexpr int kCvtA = kCvtKQ + kTC * QMAX * 4;
  static constexpr int kCvtKt = kCvtA + (CHG ? kTC * kKP * 4 : 0);
  static constexpr int kCvtV = kCvtKt + (CHG ? kTC * kKP * 4 : 0);  // CONV: post-convolution v [kTC][DV]
  static constexpr int kCvtBytes = kCvtV + (CONV ? kTC * DV * 4 : 0);
  static constexpr int kOffCvt = 2 * kRawBytes;
  static constexpr int kOffOnes = kOffCvt + 2 * kCvtBytes;  // kda: kKP ones (no pending decay)
  // CONV: the unit's weights [2 DK + DV][W] and the last W - 1 raw inputs [W - 1][2 DK + DV]
  static constexpr int kCH = 2 * DK + DV;
  static constexpr int kOffConvW = kOffOnes + (CHG ? kKP * 4 : 0);
  static constexpr int kOffCarry = kOffConvW + (CONV ? kCH * kMaxConvWidth * 4 : 0);
  static constexpr int kSmem = kOffCarry + (CONV ? (kCH * (kMaxConvWidth - 1) * kIB + 15) / 16 * 16 : 0);

  static_assert(kC == 2 || kC == 4, "columns per lane");
  static_assert(DK % (4 * kLG) == 0, "rows per lane must be a multiple of 4");
  static_assert(DV % kC == 0 && (DV >= kWarpCols ? DV % kWarpCols == 0 : kWarpCols % DV == 0),
                "columns must tile the warps");
  static_assert((DK * kIB) % 16 == 0 && (DV * kIB) % 16 == 0, "16-byte staging");
  static_assert(kRawBytes % 16 == 0 && kCvtBytes % 16 == 0, "alignment of staging buffers");
};

template <int RULE, int DK, int DV, typename IT, int MIN_BLOCKS, bool CKPT, bool QGRP, bool CONV = false>
__global__ void __launch_bounds__(
    ScanCfg<DK, DV, IT, Rule<RULE>::kChannelGate, QGRP ? kMaxQueryGroup : 1, CONV>::kThreads, MIN_BLOCKS)
    scan_kernel(const ScanParams p) {
  constexpr bool CHG = Rule<RULE>::kChannelGate;
  constexpr int QM = QGRP ? kMaxQueryGroup : 1;
  using C = ScanCfg<DK, DV, IT, CHG, QM, CONV>;
  static_assert(!(CONV && (QGRP || CKPT)), "the convolution runs in the plain scan");
  constexpr int CH = C::kCH;
  const int qg = QGRP ? p.q_group : 1;
  constexpr int R = C::kR;
  constexpr int KC = C::kC;
  extern __shared__ __align__(128) unsigned char smem[];
  float* wconv = reinterpret_cast<float*>(smem + C::kOffConvW);  // CONV
  IT* carry = reinterpret_cast<IT*>(smem + C::kOffCarry);          // CONV

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rg = lane & 3;   // row group
  const int cg = lane >> 2;  // column group within the warp
  const int col0 = warp * C::kWarpCols + cg * KC;
  const bool col_active = col0 < DV;
  const int H = p.n_v_heads;
  const int ratio = H / p.n_qk_heads;
  const int64_t units = (int64_t)p.n_seqs * H;
  const int64_t G = gridDim.x;

  const IT* qgl = static_cast<const IT*>(p.q);
  const IT* kg = static_cast<const IT*>(p.k);
  const IT* vg = static_cast<const IT*>(p.v);
  IT* og = static_cast<IT*>(p.o);
  const float* ones = reinterpret_cast<const float*>(smem + C::kOffOnes);
  if (CHG) {
    for (int i = tid; i < C::kKP; i += C::kThreads) reinterpret_cast<float*>(smem + C::kOffOnes)[i] = 1.0f;
    __syncthreads();
  }

#pragma unroll 1
  for (int64_t round = 0; round * G < units; ++round) {
    const int64_t u = round * G + ((round & 1) ? (G - 1 - blockIdx.x) : blockIdx.x);
    if (u >= units) continue;
    const int64_t si = u / H;
    const int h = (int)(u % H);
    const int hq = h / ratio;
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
    // q8 pools: the head's masks must mark exactly n_hp rows, or the row ranks leave the tile
    {
      int cs = p.src_n_hp, cd = p.dst_n_hp;
      for (int w = 0; w < DK / 32; ++w) {
        if (p.read_slot && p.src_dtype == LA_Q8) cs -= __popc(__ldg(p.src_mask + h * (DK / 32) + w));
        if (p.dst_dtype == LA_Q8) cd -= __popc(__ldg(p.dst_mask + h * (DK / 32) + w));
      }
      if (cs != 0 || cd != 0) {
        if (tid == 0) report(p.err, LA_DEVERR_Q8_MASK);
        continue;
      }
    }

    // ---- checkpoints of this sequence: after (j + 1) * ckpt_every tokens, j < n_ck
    int n_ck = 0, ck_base = 0;
    if (CKPT && p.ckpt_every > 0) {
      ck_base = __ldg(p.ckpt_cu + seq);
      n_ck = __ldg(p.ckpt_cu + seq + 1) - ck_base;
      const int fit = (t1 - t0) / p.ckpt_every;
      if (n_ck < 0 || n_ck > fit) {
        if (tid == 0) report(p.err, LA_DEVERR_CU_SEQLENS);
        n_ck = n_ck < 0 ? 0 : fit;
      }
    }

    // ---- initial state: rows rg*R .. rg*R+R-1, columns col0 .. col0+KC-1
    float S[R][KC];
    constexpr int NG = DV / 32;  // q8: 32-column groups per row; a warp's columns are group `warp`
    constexpr bool kQ8Layout = KC == 4 && DV % 32 == 0;  // q8 pools need whole 32-column groups
    if (p.read_slot && col_active) {
      const int64_t base = ((int64_t)rs * H + h) * (DK * DV);
      if (p.src_dtype == LA_Q8) {
        if constexpr (kQ8Layout) {
        const unsigned char* src =
            static_cast<const unsigned char*>(p.src) + ((int64_t)rs * H + h) * q8_tile_bytes(DK, DV, p.src_n_hp);
        const int n8 = DK - p.src_n_hp;
        Q8Rows<DK> rows;
        rows.init(p.src_mask + h * (DK / 32), rg * R);
#pragma unroll
        for (int m = 0; m < R; ++m) {
          int idx;
          if (rows.row(m, idx)) {
            load_f32<__nv_bfloat16, KC>(
                reinterpret_cast<const __nv_bfloat16*>(src + n8 * DV + n8 * NG * 4) + idx * DV + col0, S[m]);
          } else {
            uint32_t w[KC / 4];
#pragma unroll
            for (int x = 0; x < KC / 4; ++x) w[x] = reinterpret_cast<const uint32_t*>(src + idx * DV + col0)[x];
            q8_unpack<KC>(w, *reinterpret_cast<const float*>(src + n8 * DV + (idx * NG + warp) * 4), S[m]);
          }
        }
        }
      } else if (p.src_dtype == LA_F32) {
        const float* src = static_cast<const float*>(p.src) + base;
#pragma unroll
        for (int m = 0; m < R; ++m) load_f32<float, KC>(src + (rg * R + m) * DV + col0, S[m]);
      } else {
        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.src) + base;
#pragma unroll
        for (int m = 0; m < R; ++m) load_f32<__nv_bfloat16, KC>(src + (rg * R + m) * DV + col0, S[m]);
      }
    } else {
#pragma unroll
      for (int m = 0; m < R; ++m)
#pragma unroll
        for (int c = 0; c < KC; ++c) S[m][c] = 0.0f;
    }

    // ---- convolution: the unit's weights and its history (the last W - 1 raw inputs of
    //      every channel, oldest first: carry[j][c]) from the read slot, or zero
    const int cw = CONV ? p.conv_w : 1;
    if constexpr (CONV) {
      for (int idx = tid; idx < CH * cw; idx += C::kThreads) {
        const int c = idx / cw, j = idx % cw;
        wconv[idx] = c < DK ? __ldg(p.conv_wq + ((int64_t)hq * DK + c) * cw + j)
                   : c < 2 * DK ? __ldg(p.conv_wk + ((int64_t)hq * DK + (c - DK)) * cw + j)
                                : __ldg(p.conv_wv + ((int64_t)h * DV + (c - 2 * DK)) * cw + j);
      }
      const IT* hs = static_cast<const IT*>(p.conv_src) + ((int64_t)rs * H + h) * CH * (cw - 1);
      for (int idx = tid; idx < CH * (cw - 1); idx += C::kThreads) {
        const int c = idx / (cw - 1), j = idx % (cw - 1);
        if (p.read_slot) carry[j * CH + c] = hs[idx];
        else io_store(carry + j * CH + c, 0.0f);
      }
      __syncthreads();
    }

    // ---- token loop
    const int n_tok = t1 - t0;
    const int n_chunks = (n_tok + C::kTC - 1) / C::kTC;
    float gam = 1.0f;       // S = gam * St  (the registers hold St)
    float up[KC];           // pending update  St <- St + kp up^T
#pragma unroll
    for (int c = 0; c < KC; ++c) up[c] = 0.0f;
    const float* kp = nullptr;  // pending key (padded FP32 row block); nullptr: none
    const float* ap = nullptr;  // kda: pending decays (same layout); nullptr: none
    int ck_j = 0, ck_left = p.ckpt_every;  // next checkpoint, tokens until it

    // stores gam * St (the state) to slot `slot` of the destination pool
    auto store_state = [&](int slot) {
      if (!col_active) return;
      const int64_t base = ((int64_t)slot * H + h) * (DK * DV);
      if (p.dst_dtype == LA_Q8) {
        if constexpr (kQ8Layout) {
        // q8: the 8 lanes of a row group hold the row's 32-column group; its absmax is
        // reduced across them (xor 4, 8, 16) before the codes are decided
        unsigned char* dst =
            static_cast<unsigned char*>(p.dst) + ((int64_t)slot * H + h) * q8_tile_bytes(DK, DV, p.dst_n_hp);
        const int n8 = DK - p.dst_n_hp;
        Q8Rows<DK> rows;
        rows.init(p.dst_mask + h * (DK / 32), rg * R);
#pragma unroll
        for (int m = 0; m < R; ++m) {
          float y[KC];
          float amax = 0.0f;
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            y[c] = gam * S[m][c];
            amax = fmaxf(amax, fabsf(y[c]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 8));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
          int idx;
          if (rows.row(m, idx)) {
            store_f32<__nv_bfloat16, KC>(
                reinterpret_cast<__nv_bfloat16*>(dst + n8 * DV + n8 * NG * 4) + idx * DV + col0, y);
          } else {
            float sc, inv;
            q8_scales(amax, sc, inv);
            uint32_t w[KC / 4];
            q8_pack<KC>(y, inv, w);
#pragma unroll
            for (int x = 0; x < KC / 4; ++x) reinterpret_cast<uint32_t*>(dst + idx * DV + col0)[x] = w[x];
            if (cg == 0) *reinterpret_cast<float*>(dst + n8 * DV + (idx * NG + warp) * 4) = sc;
          }
        }
        }
      } else if (p.dst_dtype == LA_F32) {
        float* dst = static_cast<float*>(p.dst) + base;
#pragma unroll
        for (int m = 0; m < R; ++m) {
          float y[KC];
#pragma unroll
          for (int c = 0; c < KC; ++c) y[c] = gam * S[m][c];
          store_f32<float, KC>(dst + (rg * R + m) * DV + col0, y);
        }
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dst) + base;
#pragma unroll
        for (int m = 0; m < R; ++m) {
          float y[KC];
#pragma unroll
          for (int c = 0; c < KC; ++c) y[c] = gam * S[m][c];
          store_f32<__nv_bfloat16, KC>(dst + (rg * R + m) * DV + col0, y);
        }
      }
    };

    // applies the pending update St <- (alpha .) St + kp up^T and clears it
    auto apply_pending = [&]() {
#pragma unroll
      for (int m4 = 0; m4 < R / 4; ++m4) {
        const float4 k4p = *reinterpret_cast<const float4*>(kp + 4 * m4);
        float4 a4p = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        if (CHG && ap) a4p = *reinterpret_cast<const float4*>(ap + 4 * m4);
        const float kpv[4] = {k4p.x, k4p.y, k4p.z, k4p.w};
        const float apv[4] = {a4p.x, a4p.y, a4p.z, a4p.w};
#pragma unroll
        for (int mm = 0; mm < 4; ++mm)
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            float& x = S[4 * m4 + mm][c];
            x = CHG ? fmaf(kpv[mm], up[c], apv[mm] * x) : fmaf(kpv[mm], up[c], x);
          }
      }
#pragma unroll
      for (int c = 0; c < KC; ++c) up[c] = 0.0f;
    };

    auto issue = [&](int ch) {
      unsigned char* raw = smem + (ch & 1) * C::kRawBytes;
      const int tok0 = t0 + ch * C::kTC;
      const int n = (t1 - tok0) < C::kTC ? (t1 - tok0) : C::kTC;
      for (int idx = tid; idx < n * C::kQKVecs; idx += C::kThreads) {
        const int tt = idx / C::kQKVecs, pc = idx % C::kQKVecs;
        const int64_t row = ((int64_t)(tok0 + tt) * p.n_qk_heads + hq) * DK;
        cp_async_16(raw + C::kRawK + (tt * DK) * C::kIB + pc * 16,
                    reinterpret_cast<const unsigned char*>(kg + row) + pc * 16);
      }
      // query rows: the q/k head's, or the qg consecutive query heads of this state head
      for (int idx = tid; idx < n * qg * C::kQKVecs; idx += C::kThreads) {
        const int tq = idx / C::kQKVecs, pc = idx % C::kQKVecs;
        const int tt = tq / qg, qi = tq % qg;
        const int64_t row = QGRP ? ((int64_t)(tok0 + tt) * H * qg + (int64_t)h * qg + qi) * DK
                                 : ((int64_t)(tok0 + tt) * p.n_qk_heads + hq) * DK;
        cp_async_16(raw + C::kRawQ + ((tt * QM + qi) * DK) * C::kIB + pc * 16,
                    reinterpret_cast<const unsigned char*>(qgl + row) + pc * 16);
      }
      for (int idx = tid; idx < n * C::kVVecs; idx += C::kThreads) {
        const int tt = idx / C::kVVecs, pc = idx % C::kVVecs;
        const int64_t row = ((int64_t)(tok0 + tt) * H + h) * DV;
        cp_async_16(raw + C::kRawV + (tt * DV) * C::kIB + pc * 16,
                    reinterpret_cast<const unsigned char*>(vg + row) + pc * 16);
      }
      for (int tt = tid; tt < n; tt += C::kThreads) {
        const int64_t gi = (int64_t)(tok0 + tt) * H + h;
        if (Rule<RULE>::kUsesGate) cp_async_4(raw + C::kRawG + tt * 4, p.g + gi);
        if (Rule<RULE>::kUsesBeta) cp_async_4(raw + C::kRawB + tt * 4, p.beta + gi);
      }
      if (CHG) {
        constexpr int kAVecs = DK / 4;  // 16-byte pieces of one token's decays
        for (int idx = tid; idx < n * kAVecs; idx += C::kThreads) {
          const int tt = idx / kAVecs, pc = idx % kAVecs;
          cp_async_16(raw + C::kRawA + tt * DK * 4 + pc * 16, p.g + ((int64_t)(tok0 + tt) * H + h) * DK + 4 * pc);
        }
      }
      cp_async_commit();
    };

    if (n_chunks > 0) issue(0);
#pragma unroll 1
    for (int ch = 0; ch < n_chunks; ++ch) {
      const int buf = ch & 1;
      if (ch + 1 < n_chunks) {
        issue(ch + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();

      const unsigned char* raw = smem + buf * C::kRawBytes;
      unsigned char* cvt = smem + C::kOffCvt + buf * C::kCvtBytes;
      float* kf = reinterpret_cast<float*>(cvt + C::kCvtK);
      float* qf = reinterpret_cast<float*>(cvt + C::kCvtQ);
      float* kqs = reinterpret_cast<float*>(cvt + C::kCvtKQ);
      const IT* kraw = reinterpret_cast<const IT*>(raw + C::kRawK);
      const IT* qraw = reinterpret_cast<const IT*>(raw + C::kRawQ);
      const int tok0 = t0 + ch * C::kTC;
      const int n = (t1 - tok0) < C::kTC ? (t1 - tok0) : C::kTC;

      float* af = reinterpret_cast<float*>(cvt + C::kCvtA);
      float* ktf = reinterpret_cast<float*>(cvt + C::kCvtKt);
      float* vf = reinterpret_cast<float*>(cvt + C::kCvtV);
      if constexpr (CONV) {
        // the convolution: a thread per channel walks the chunk's tokens with the window of
        // its W - 1 previous inputs in registers (starting from the carried ones), and leaves
        // the chunk's last W - 1 inputs as the new carried window of its channel
        const IT* vraw_in = reinterpret_cast<const IT*>(raw + C::kRawV);
        for (int c = tid; c < CH; c += C::kThreads) {
          float w[kMaxConvWidth], win[kMaxConvWidth - 1];
#pragma unroll
          for (int j = 0; j < kMaxConvWidth; ++j) w[j] = j < cw ? wconv[c * cw + j] : 0.0f;
          float wnew = 0.0f;  // the newest input's weight, w[cw - 1] (kept out of dynamic indexing)
#pragma unroll
          for (int j = 0; j < kMaxConvWidth; ++j)
            if (j == cw - 1) wnew = w[j];
#pragma unroll
          for (int j = 0; j < kMaxConvWidth - 1; ++j) win[j] = j < cw - 1 ? io_load(carry + j * CH + c) : 0.0f;
          const int i = c % DK;
          const int prow = (i / R) * C::kRowStride + (i % R);
          const IT* src = c < DK ? qraw + c : c < 2 * DK ? kraw + (c - DK) : vraw_in + (c - 2 * DK);
          const int sstride = c < DK ? QM * DK : c < 2 * DK ? DK : DV;
          float* dst = c < DK ? qf + prow : c < 2 * DK ? kf + prow : vf + (c - 2 * DK);
          const int dstride = c < DK ? QM * C::kKP : c < 2 * DK ? C::kKP : DV;
          for (int tt = 0; tt < n; ++tt) {
            const float x = io_load(src + tt * sstride);
            float y = wnew * x;
#pragma unroll
            for (int j = 0; j < kMaxConvWidth - 1; ++j)
              if (j < cw - 1) y = fmaf(w[j], win[j], y);
#pragma unroll
            for (int j = 0; j < kMaxConvWidth - 1; ++j)
              win[j] = j < cw - 2 ? win[j + 1] : (j == cw - 2 ? x : win[j]);
            if (p.conv_act) y = __fdividef(y, 1.0f + __expf(-y));
            dst[tt * dstride] = y;
          }
#pragma unroll
          for (int j = 0; j < kMaxConvWidth - 1; ++j)
            if (j < cw - 1) io_store(carry + j * CH + c, win[j]);
        }
        if (CHG) {
          for (int idx = tid; idx < n * DK; idx += C::kThreads) {
            const int tt = idx / DK, i = idx % DK;
            af[tt * C::kKP + (i / R) * C::kRowStride + (i % R)] = reinterpret_cast<const float*>(raw + C::kRawA)[idx];
          }
        }
        __syncthreads();
        // per token: unit length for q and k (when asked), k.q, the decayed rows (kda)
        for (int tt = warp; tt < n; tt += C::kWarps) {
          float sq = 0.0f, sk = 0.0f, d = 0.0f;
          for (int i = lane; i < DK; i += 32) {
            const int pi = tt * C::kKP + (i / R) * C::kRowStride + (i % R);
            const float qv = qf[tt * QM * C::kKP + (i / R) * C::kRowStride + (i % R)], kv = kf[pi];
            sq = fmaf(qv, qv, sq);
            sk = fmaf(kv, kv, sk);
            d = fmaf(kv, qv, d);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            d += __shfl_xor_sync(0xffffffffu, d, off);
          }
          const float rq = p.conv_l2norm ? rsqrtf(sq + 1e-6f) : 1.0f;
          const float rk = p.conv_l2norm ? rsqrtf(sk + 1e-6f) : 1.0f;
          for (int i = lane; i < DK; i += 32) {
            const int pi = tt * C::kKP + (i / R) * C::kRowStride + (i % R);
            const int qi_ = tt * QM * C::kKP + (i / R) * C::kRowStride + (i % R);
            const float kv = kf[pi] * rk;
            kf[pi] = kv;
            qf[qi_] = CHG ? qf[qi_] * rq * af[pi] : qf[qi_] * rq;
            if (CHG) ktf[pi] = af[pi] * kv;
          }
          if (lane == 0) kqs[tt * QM] = d * rq * rk;
        }
      } else {
      // convert keys / queries to padded FP32, and k.q per token (kda: also the decays,
      // the decayed key and the decayed query)
      for (int idx = tid; idx < n * DK; idx += C::kThreads) {
        const int tt = idx / DK, i = idx % DK;
        const int pi = tt * C::kKP + (i / R) * C::kRowStride + (i % R);
        const float kx = io_load(kraw + idx);
        kf[pi] = kx;
        if (CHG) {
          const float ax = reinterpret_cast<const float*>(raw + C::kRawA)[idx];
          af[pi] = ax;
          ktf[pi] = ax * kx;
        }
      }
      for (int idx = tid; idx < n * qg * DK; idx += C::kThreads) {
        const int tq = idx / DK, i = idx % DK;
        const int tt = tq / qg, qi = tq % qg;
        const int pi = (tt * QM + qi) * C::kKP + (i / R) * C::kRowStride + (i % R);
        const float qx = io_load(qraw + (tt * QM + qi) * DK + i);
        qf[pi] = CHG ? reinterpret_cast<const float*>(raw + C::kRawA)[tt * DK + i] * qx : qx;
      }
      for (int tq = warp; tq < n * qg; tq += C::kWarps) {
        const int tt = tq / qg, qi = tq % qg;
        float d = 0.0f;
        for (int i = lane; i < DK; i += 32)
          d = fmaf(io_load(kraw + tt * DK + i), io_load(qraw + (tt * QM + qi) * DK + i), d);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        if (lane == 0) kqs[tt * QM + qi] = d;
      }
      }
      __syncthreads();

      const IT* vraw = reinterpret_cast<const IT*>(raw + C::kRawV);
      const float* graw = reinterpret_cast<const float*>(raw + C::kRawG);
      const float* braw = reinterpret_cast<const float*>(raw + C::kRawB);
#pragma unroll 1
      for (int tt = 0; tt < n; ++tt) {
        const float* kc = kf + tt * C::kKP + rg * C::kRowStride;
        const float* qc = qf + tt * QM * C::kKP + rg * C::kRowStride;
        const float* ksum = CHG ? ktf + tt * C::kKP + rg * C::kRowStride : kc;  // key of S^T k
        const float* kpp = kp ? kp : kc;  // no pending update before the first token
        const float* apc = ap ? ap : ones + rg * C::kRowStride;  // kda: pending decays
        float pa[KC], ra[KC], pb[KC], rb2[KC];  // even / odd row partial sums
#pragma unroll
        for (int c = 0; c < KC; ++c) pa[c] = ra[c] = pb[c] = rb2[c] = 0.0f;
#pragma unroll
        for (int m4 = 0; m4 < R / 4; ++m4) {
          const float4 k4p = *reinterpret_cast<const float4*>(kpp + 4 * m4);
          const float4 k4 = *reinterpret_cast<const float4*>(ksum + 4 * m4);
          const float4 q4 = *reinterpret_cast<const float4*>(qc + 4 * m4);
          float4 a4p = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
          if (CHG) a4p = *reinterpret_cast<const float4*>(apc + 4 * m4);
          const float kpv[4] = {k4p.x, k4p.y, k4p.z, k4p.w};
          const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
          const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
          const float apv[4] = {a4p.x, a4p.y, a4p.z, a4p.w};
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) {
#pragma unroll
            for (int c = 0; c < KC; ++c) {
              float& x = S[4 * m4 + mm][c];
              x = CHG ? fmaf(kpv[mm], up[c], apv[mm] * x) : fmaf(kpv[mm], up[c], x);
              if (mm & 1) {
                if (Rule<RULE>::kPredicts) pb[c] = fmaf(x, kv[mm], pb[c]);
                rb2[c] = fmaf(x, qv[mm], rb2[c]);
              } else {
                if (Rule<RULE>::kPredicts) pa[c] = fmaf(x, kv[mm], pa[c]);
                ra[c] = fmaf(x, qv[mm], ra[c]);
              }
            }
          }
        }
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          pa[c] += pb[c];
          ra[c] += rb2[c];
          if (Rule<RULE>::kPredicts) {
            pa[c] += __shfl_xor_sync(0xffffffffu, pa[c], 1);
            pa[c] += __shfl_xor_sync(0xffffffffu, pa[c], 2);
          }
          ra[c] += __shfl_xor_sync(0xffffffffu, ra[c], 1);
          ra[c] += __shfl_xor_sync(0xffffffffu, ra[c], 2);
        }
        const float gt = Rule<RULE>::kUsesGate ? graw[tt] : 1.0f;
        const float bt = Rule<RULE>::kUsesBeta ? braw[tt] : 1.0f;
        float a, bcoef, cdel;
        Rule<RULE>::coeffs(gt, bt, a, bcoef, cdel);
        const float kq = kqs[tt * QM];
        float vv[KC];
#pragma unroll
        for (int c = 0; c < KC; ++c) vv[c] = 0.0f;
        if (col_active) {
          if constexpr (CONV) load_f32<float, KC>(vf + tt * DV + col0, vv);
          else load_f32<IT, KC>(vraw + tt * DV + col0, vv);
        }
        // u = b (v - c S^T k),  o = scale (a S^T q + (k.q) u),  with S = gam St
        float uu[KC], oc[KC];
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          uu[c] = bcoef * (vv[c] - cdel * (gam * pa[c]));
          oc[c] = p.scale * fmaf(a, gam * ra[c], kq * uu[c]);
        }
        // o row of the token's first query
        const int64_t orow = QGRP ? ((int64_t)(tok0 + tt) * H + h) * qg : (int64_t)(tok0 + tt) * H + h;
        if (col_active && rg < KC) {
          float mine = oc[0];
#pragma unroll
          for (int c = 1; c < KC; ++c) mine = (rg == c) ? oc[c] : mine;
          io_store(og + orow * DV + col0 + rg, mine);
        }
        // the other queries of the group: o = scale (a S^T q + (k.q) u) from the same registers
        if (QGRP) {
#pragma unroll 1
          for (int qi = 1; qi < qg; ++qi) {
            const float* qci = qc + qi * C::kKP;
            float ea[KC], eb[KC];
#pragma unroll
            for (int c = 0; c < KC; ++c) ea[c] = eb[c] = 0.0f;
#pragma unroll
            for (int m4 = 0; m4 < R / 4; ++m4) {
              const float4 q4 = *reinterpret_cast<const float4*>(qci + 4 * m4);
              const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
              for (int mm = 0; mm < 4; ++mm)
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                  if (mm & 1) eb[c] = fmaf(S[4 * m4 + mm][c], qv[mm], eb[c]);
                  else ea[c] = fmaf(S[4 * m4 + mm][c], qv[mm], ea[c]);
                }
            }
            const float kqi = kqs[tt * QM + qi];
            float oi[KC];
#pragma unroll
            for (int c = 0; c < KC; ++c) {
              float rr = ea[c] + eb[c];
              rr += __shfl_xor_sync(0xffffffffu, rr, 1);
              rr += __shfl_xor_sync(0xffffffffu, rr, 2);
              oi[c] = p.scale * fmaf(a, gam * rr, kqi * uu[c]);
            }
            if (col_active && rg < KC) {
              float mine = oi[0];
#pragma unroll
              for (int c = 1; c < KC; ++c) mine = (rg == c) ? oi[c] : mine;
              io_store(og + (orow + qi) * DV + col0 + rg, mine);
            }
          }
        }
        // S_t = a S_{t-1} + k u^T:  gam <- a gam,  St <- St + k (u / gam)^T (applied in
        // the next token's pass).  A gate product outside [2^-40, 2^40] is folded now:
        // the registers hold St_{t-1}, so St <- (a gam) St and gam <- 1.
        if (Rule<RULE>::kUsesGate) {
          const float gnew = a * gam;
          if (!(fabsf(gnew) >= 0x1p-40f && fabsf(gnew) <= 0x1p40f)) {
#pragma unroll
            for (int m = 0; m < R; ++m)
#pragma unroll
              for (int c = 0; c < KC; ++c) S[m][c] *= gnew;
            gam = 1.0f;
          } else {
            gam = gnew;
          }
          const float inv = __fdividef(1.0f, gam);
#pragma unroll
          for (int c = 0; c < KC; ++c) up[c] = uu[c] * inv;
        } else {
#pragma unroll
          for (int c = 0; c < KC; ++c) up[c] = uu[c];
        }
        kp = kc;
        if (CHG) ap = af + tt * C::kKP + rg * C::kRowStride;
        if (CKPT && ck_j < n_ck && --ck_left == 0) {
          // checkpoint: apply this token's update now and store the state
          ck_left = p.ckpt_every;
          apply_pending();
          kp = nullptr;
          ap = nullptr;
          const int cs = __ldg(p.ckpt_slots + ck_base + ck_j);
          if (cs >= 0 && cs < p.dst_slots) {
            store_state(cs);
          } else if (tid == 0) {
            report(p.err, LA_DEVERR_WRITE_SLOT);
          }
          ++ck_j;
        }
      }
      __syncthreads();
    }

    // ---- last pending update, store the final state (and the convolution history)
    if (kp) apply_pending();
    store_state(ws);
    if constexpr (CONV) {
      IT* hd = static_cast<IT*>(p.conv_dst) + ((int64_t)ws * H + h) * CH * (cw - 1);
      for (int idx = tid; idx < CH * (cw - 1); idx += C::kThreads) {
        const int c = idx / (cw - 1), j = idx % (cw - 1);
        hd[idx] = carry[j * CH + c];
      }
    }
    // the next unit's staging must not overwrite what this unit still reads
    __syncthreads();
  }
}

template <int RULE, int DK, int DV, typename IT, bool QGRP, bool CONV = false>
cudaError_t launch_scan(const ScanParams& p, cudaStream_t stream) {
  using C = ScanCfg<DK, DV, IT, Rule<RULE>::kChannelGate, QGRP ? kMaxQueryGroup : 1, CONV>;
  if constexpr (CONV) {
    constexpr int kMinBlocks = LA_SCAN_MIN_BLOCKS_CONV;
    const void* fn = reinterpret_cast<const void*>(&scan_kernel<RULE, DK, DV, IT, kMinBlocks, false, false, true>);
    const int per_sm = prepare_kernel(fn, C::kThreads, C::kSmem);
    if (per_sm <= 0) return cudaErrorInvalidConfiguration;
    const int64_t units = (int64_t)p.n_seqs * p.n_v_heads;
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int grid = (int)(units < cap ? units : cap);
    scan_kernel<RULE, DK, DV, IT, kMinBlocks, false, false, true><<<grid, C::kThreads, C::kSmem, stream>>>(p);
    return cudaGetLastError();
  }
  constexpr int kMinBlocks = LA_SCAN_MIN_BLOCKS;
  constexpr int kMinBlocksCk = LA_SCAN_MIN_BLOCKS_CKPT;
  // checkpoints are a separate instantiation so that the plain scan's loop carries no
  // checkpoint bookkeeping (the query-group direction has none)
  const bool ck = !QGRP && p.ckpt_every > 0;
  const void* fn = ck ? reinterpret_cast<const void*>(&scan_kernel<RULE, DK, DV, IT, kMinBlocksCk, !QGRP, QGRP>)
                      : reinterpret_cast<const void*>(&scan_kernel<RULE, DK, DV, IT, kMinBlocks, false, QGRP>);
  const int per_sm = prepare_kernel(fn, C::kThreads, C::kSmem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  const int64_t units = (int64_t)p.n_seqs * p.n_v_heads;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)(units < cap ? units : cap);
  if (ck)
    scan_kernel<RULE, DK, DV, IT, kMinBlocksCk, !QGRP, QGRP><<<grid, C::kThreads, C::kSmem, stream>>>(p);
  else
    scan_kernel<RULE, DK, DV, IT, kMinBlocks, false, QGRP><<<grid, C::kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

template <typename IT, bool QGRP>
ScanLaunchFn find_scan_impl(int rule, int dk, int dv) {
#define LA_SCAN_CASE(R, K, V) \
  if (rule == R && dk == K && dv == V) return &launch_scan<R, K, V, IT, QGRP>;
#define LA_SCAN_SHAPES(R) LA_SCAN_CASE(R, 16, 16) LA_SCAN_CASE(R, 64, 64) LA_SCAN_CASE(R, 128, 64) LA_SCAN_CASE(R, 128, 128)
  LA_SCAN_SHAPES(LA_RULE_LINEAR)
  LA_SCAN_SHAPES(LA_RULE_GATED)
  LA_SCAN_SHAPES(LA_RULE_DELTA)
  LA_SCAN_SHAPES(LA_RULE_GATED_DELTA)
  LA_SCAN_SHAPES(LA_RULE_KDA)
#undef LA_SCAN_SHAPES
#undef LA_SCAN_CASE
  return nullptr;
}

// Launcher table of the scan with the convolution ahead (io dtype IT).
template <typename IT>
ScanLaunchFn find_scan_conv_impl(int rule, int dk, int dv) {
#define LA_SCONV_CASE(R, K, V) \
  if (rule == R && dk == K && dv == V) return &launch_scan<R, K, V, IT, false, true>;
#define LA_SCONV_SHAPES(R) LA_SCONV_CASE(R, 16, 16) LA_SCONV_CASE(R, 64, 64) LA_SCONV_CASE(R, 128, 64) LA_SCONV_CASE(R, 128, 128)
  LA_SCONV_SHAPES(LA_RULE_LINEAR)
  LA_SCONV_SHAPES(LA_RULE_GATED)
  LA_SCONV_SHAPES(LA_RULE_DELTA)
  LA_SCONV_SHAPES(LA_RULE_GATED_DELTA)
  LA_SCONV_SHAPES(LA_RULE_KDA)
#undef LA_SCONV_SHAPES
#undef LA_SCONV_CASE
  return nullptr;
}

}  // namespace la
