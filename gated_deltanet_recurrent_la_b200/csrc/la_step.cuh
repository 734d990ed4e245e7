// la_step.cuh -- batched decode step (one token per request) on sm_100a.
//
// The operation is the recurrent-state update of the "Gated DeltaNet" glossary page
// (Technical definition) under the four update rules of the ONNX LinearAttention
// operator ("Seven Architectures Replacing KV Cache With Bounded Mutable State", section
// "ONNX LinearAttention / FlashInfer"):  u = b (v - c S^T k),  S' = a S + k u^T,
// o = scale S'^T q, computed in the rearranged form of the "Gated DeltaNet" page
// (Engineering details)  o = scale (a S^T q + (k.q) u)  so one pass over S serves both
// the update and the readout.  The state is read from and written to HBM once per
// step, which makes the step HBM-bound (about one flop per byte; "SSM / linear-RNN
// decode: the constant-size recurrent state update").
//
// Design (B200):
//  * persistent CTAs, one per SM (the ring of stages fills most of the 227 KB of shared
//    memory), each walking tiles t = blockIdx.x + i * gridDim.x, tile t = (request
//    t / H_v, head t % H_v);
//  * warp specialisation: one producer warp streams each whole d_k x d_v state tile (a
//    contiguous 8-64 KiB block of the pool) plus q, k, v into a shared-memory stage
//    with 1-D bulk copies on the TMA engine, signalling an mbarrier -- the
//    asynchronous movement of the state named on the "Gated DeltaNet" page (How to read it) --
//    so that several tiles are in flight per SM at all times;
//  * every column of S evolves on its own, so each consumer warp owns a strip of up to
//    32 columns of a tile for all d_k rows and needs nobody else: lanes split the strip
//    into 16-byte column chunks x row blocks, hold the strip's 128 state values in FP32
//    registers, finish S^T k and S^T q with xor-shuffles inside the warp, form u and o,
//    release the stage on their own, and store the new state with 16-byte stores.
//    Warps of different tiles run concurrently; there is no CTA-wide barrier.  Four
//    consumer warps (plus the producer) keep every SM sub-partition at <= 2 warps so a
//    thread may hold its 128 state values without spilling.
//  * the channel-wise gate of Kimi Delta Attention ("Seven Architectures ...", section
//    "Kimi Linear") keeps every column independent: the d_k decays ride in the stage
//    with the tile and scale the keys of the two reductions and the rows of the update.
//  * FP32 arithmetic in pairs (packed FFMA2 / FMUL2 only where it measures faster).
#pragma once

#include <cstdint>
#include <type_traits>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {

constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

struct StepMeta {
  float g;
  float beta;
  int32_t valid;
  int32_t ws;       // write slot (the convolution history goes there too)
  int64_t dst_off;  // byte offset of the destination tile in the destination pool
  int64_t o_off;    // element offset of o[b, h, 0]
};

// Consumer warps per CTA and the widest column strip of one warp.  With 4 consumer
// warps plus the producer no SM sub-partition holds more than 2 warps, so a thread may
// use up to 255 registers (a strip of 32 x 128 holds 128 FP32 state values per lane).
#ifndef LA_STEP_CONSUMER_WARPS
#define LA_STEP_CONSUMER_WARPS 4
#endif
#ifndef LA_STEP_STRIP_COLS
#define LA_STEP_STRIP_COLS 32
#endif
// Launch with programmatic stream serialization so that a step's prologue overlaps the
// tail of the previous kernel on the stream.
#ifndef LA_STEP_PDL
#define LA_STEP_PDL 1
#endif

// CHG: the rule carries a channel-wise gate (kda), d_k FP32 decays staged with the tile.
// QMAX: query rows a stage holds (1, or kMaxQueryGroup in the query-group direction).
// CONV: the short causal convolution runs ahead of the step (the stage also holds the
// tile's convolution history and weights, and a scratch of its post-convolution q, k, v).
template <int DK, int DV, typename ST, typename IT, bool CHG = false, int QMAX = 1, bool CONV = false>
struct StepCfg {
  static constexpr bool kQ8 = std::is_same<ST, q8_t>::value;
  static constexpr int kSB = kQ8 ? 2 : (int)sizeof(ST);  // (q8: the BF16 rows' lane layout)
  static constexpr int kVec = 16 / kSB;                  // state elements per lane and row
  static constexpr int kCW = DV < LA_STEP_STRIP_COLS ? DV : LA_STEP_STRIP_COLS;  // strip width
  static constexpr int kWPT = DV / kCW;                 // warps per tile
  static constexpr int kNCH = kCW / kVec;               // 16-byte chunks per strip row
  static constexpr int kRG = 32 / kNCH;                 // row blocks per warp
  static constexpr int kRL = DK / kRG;                  // rows per lane
  static constexpr int kConsumerWarps = kWPT > LA_STEP_CONSUMER_WARPS ? kWPT : LA_STEP_CONSUMER_WARPS;
  static constexpr int kTeams = kConsumerWarps / kWPT;  // tiles in compute at once
  // CONV: three warps (the q, k and v channels) run the convolution ahead of the consumers
  static constexpr int kConvWarps = CONV ? 3 : 0;
  static constexpr int kProducerWarp = kConsumerWarps + kConvWarps;
  static constexpr int kThreads = (kProducerWarp + 1) * 32;
  // stage room for one tile; q8 tiles hold at most DK / 4 BF16 rows
  static constexpr int kTileBytes = kQ8 ? (int)q8_tile_bytes(DK, DV, DK / 4) : DK * DV * kSB;
  static constexpr int kQKBytes = DK * (int)sizeof(IT);
  static constexpr int kVBytes = DV * (int)sizeof(IT);
  static constexpr int kGBytes = CHG ? DK * 4 : 0;
  // stage layout: tile | QMAX query rows | key | v | decays (kda)
  static constexpr int kOffK = kTileBytes + QMAX * kQKBytes;
  static constexpr int kOffV = kOffK + kQKBytes;
  static constexpr int kOffA = kOffV + kVBytes;
  static constexpr int kOffHist = kOffA + kGBytes;
  static constexpr int kHistBytes = CONV ? (2 * DK + DV) * (kMaxConvWidth - 1) * (int)sizeof(IT) : 0;
  static constexpr int kOffConvW = kOffHist + kHistBytes;   // the tile's weights [q | k | v channels][W]
  static constexpr int kConvWBytes = CONV ? (2 * DK + DV) * kMaxConvWidth * 4 : 0;
  static constexpr int kCopyBytes = kOffConvW + kConvWBytes;  // with all QMAX query rows, widest convolution
  static constexpr int kStageBytes = round_up(kCopyBytes, 128);
  // CONV, per stage: the tile's post-convolution q | k | v (FP32)
  static constexpr int kScrFloats = CONV ? 2 * DK + DV : 0;
  static constexpr int kStages = CONV ? cmax(2, cmin(12, (222 * 1024) / (kStageBytes + kScrFloats * 4)))
                                      : cmax(2, cmin(12, (204 * 1024) / kStageBytes));
  static constexpr int kOffMeta = kStages * kStageBytes;
  static constexpr int kOffBars = round_up(kOffMeta + kStages * (int)sizeof(StepMeta), 8);
  // barriers per stage: full, empty (and CONV: convolution done)
  static constexpr int kOffScratch = round_up(kOffBars + (CONV ? 3 : 2) * kStages * 8, 16);
  static constexpr int kSmem = kOffScratch + kStages * kScrFloats * 4;

  static_assert(kNCH >= 1 && kNCH <= 32 && (32 % kNCH) == 0, "strip row must map onto a power-of-two lane group");
  static_assert(kRL >= 1 && DK % kRG == 0, "rows must split evenly over the row blocks");
  static_assert(kConsumerWarps % kWPT == 0, "whole tiles per team");
  static_assert(kQKBytes % 16 == 0 && kVBytes % 16 == 0 && kTileBytes % 16 == 0 && kGBytes % 16 == 0,
                "bulk copies move 16-byte units");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// The convolution warps of a CONV step CTA: warp cw takes the q (cw = 0), k (1) or v (2)
// channels of every tile of the CTA, in order, as soon as its stage has arrived.  Channel c
// is y = sum_j w[c][j] x_{t-W+1+j} over the W - 1 staged history inputs and the current
// input (weights staged with the tile), then SiLU when asked; q and k are then scaled to
// unit length when asked (a warp reduction: one warp holds all of q's or k's channels).
// The results land in the stage's FP32 scratch, the channels' new histories (the last
// W - 1 inputs) go to the tile's write slot, and the warp arrives on the stage's
// convolution barrier, which the consumers wait for.  Skipped tiles only arrive.
template <int DK, int DV, typename IT, typename C>
__device__ __forceinline__ void conv_group(const StepParams& p, unsigned char* smem, const StepMeta* meta,
                                           uint64_t* full, uint64_t* conv_done, int64_t n_my, int cw, int lane) {
  constexpr int CH = 2 * DK + DV;
  constexpr int kPer = ((DK > DV ? DK : DV) + 31) / 32;  // channels per lane
  const int H = p.n_v_heads;
  const int W = p.conv_w;
  const int c_beg = cw == 0 ? 0 : cw == 1 ? DK : 2 * DK;
  const int n_ch = cw == 2 ? DV : DK;
  const int x_off = cw == 0 ? C::kTileBytes : cw == 1 ? C::kOffK : C::kOffV;
  for (int64_t it = 0; it < n_my; ++it) {
    const int stage = (int)(it % C::kStages);
    const uint32_t round = (uint32_t)(it / C::kStages);
    if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], round & 1u, p.wait_ns))) {
      if (lane == 0) report(p.err, LA_DEVERR_TIMEOUT);
      return;
    }
    const StepMeta m = meta[stage];
    if (m.valid) {
      const unsigned char* sb = smem + stage * C::kStageBytes;
      const IT* x = reinterpret_cast<const IT*>(sb + x_off);
      const IT* hist = reinterpret_cast<const IT*>(sb + C::kOffHist);
      const float* wts = reinterpret_cast<const float*>(sb + C::kOffConvW);
      float* scr = reinterpret_cast<float*>(smem + C::kOffScratch) + stage * C::kScrFloats;
      const int h = (int)((blockIdx.x + it * gridDim.x) % H);
      IT* hd = static_cast<IT*>(p.conv_dst) + ((int64_t)m.ws * H + h) * CH * (W - 1);
      float y[kPer];
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int cl = lane + 32 * i;
        y[i] = 0.0f;
        if (cl < n_ch) {
          const int c = c_beg + cl;
          const float* w = wts + c * W;
          float acc = w[W - 1] * io_load(x + cl);
#pragma unroll
          for (int j = 0; j < kMaxConvWidth - 1; ++j)
            if (j < W - 1) acc = fmaf(w[j], io_load(hist + c * (W - 1) + j), acc);
          if (p.conv_act) acc = __fdividef(acc, 1.0f + __expf(-acc));
          y[i] = acc;
          ss = fmaf(acc, acc, ss);
          for (int j = 0; j < W - 2; ++j) hd[c * (W - 1) + j] = hist[c * (W - 1) + j + 1];
          hd[c * (W - 1) + W - 2] = x[cl];
        }
      }
      float rn = 1.0f;
      if (cw < 2 && p.conv_l2norm) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        rn = rsqrtf(ss + 1e-6f);
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int cl = lane + 32 * i;
        if (cl < n_ch) scr[c_beg + cl] = y[i] * rn;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&conv_done[stage]);
  }
}

// The producer warp of a step CTA (whose stage layout is C): its lanes fetch the slot ids
// and gates of the next 32 of the CTA's tiles; lane 0 checks each tile (slots in range,
// q8 masks marking n_hp rows), writes its meta, and issues its bulk copies into the next
// free stage (the state tile with an evict-first policy), or arrives without data for a
// tile that is skipped.  A wait that runs out reports LA_DEVERR_TIMEOUT and ends the
// issue; the warp never retires with copies in flight.
template <int RULE, int DK, int DV, typename ST, typename IT, bool QGRP, bool CONV, typename C>
__device__ __forceinline__ void step_producer(const StepParams& p, unsigned char* smem, StepMeta* meta,
                                              uint64_t* full, uint64_t* empty, int64_t n_my, int lane) {
  constexpr bool CHG = Rule<RULE>::kChannelGate;
  const int H = p.n_v_heads;
  const int qg = QGRP ? p.q_group : 1;
  const uint64_t pol_stream = policy_evict_first();
  const int ratio = H / p.n_qk_heads;
  const unsigned char* src = static_cast<const unsigned char*>(p.src);
  const int tile_bytes = C::kQ8 ? (int)q8_tile_bytes(DK, DV, p.n_hp) : C::kTileBytes;
  const IT* q = static_cast<const IT*>(p.q);
  const IT* k = static_cast<const IT*>(p.k);
  const IT* v = static_cast<const IT*>(p.v);
  bool abort = false;
  int64_t issued = 0;
  for (int64_t i0 = 0; i0 < n_my && !abort; i0 += 32) {
    // lanes fetch the slot ids and gates of the next 32 tiles
    const int64_t ii = i0 + lane;
    int32_t rs = -1, ws = -1;
    float gg = 1.0f, bb = 1.0f;
    if (ii < n_my) {
      const int64_t t = blockIdx.x + ii * gridDim.x;
      const int b = (int)(t / H);
      rs = p.read_slot ? __ldg(p.read_slot + b) : b;
      ws = p.write_slot ? __ldg(p.write_slot + b) : b;
      if (Rule<RULE>::kUsesGate) gg = __ldg(p.g + t);
      if (Rule<RULE>::kUsesBeta) bb = __ldg(p.beta + t);
    }
    const int cnt = (int)((n_my - i0) < 32 ? (n_my - i0) : 32);
    for (int j = 0; j < cnt; ++j) {
      const int32_t rs_j = __shfl_sync(0xffffffffu, rs, j);
      const int32_t ws_j = __shfl_sync(0xffffffffu, ws, j);
      const float g_j = __shfl_sync(0xffffffffu, gg, j);
      const float b_j = __shfl_sync(0xffffffffu, bb, j);
      const int64_t it = i0 + j;
      const int stage = (int)(it % C::kStages);
      const uint32_t round = (uint32_t)(it / C::kStages);
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&empty[stage], (round & 1u) ^ 1u, p.wait_ns);
        if (ok && blockIdx.x == 0 && it == p.withhold) {
          // test hook: this tile's copies are never issued and its arrival never comes (its
          // consumers' waits run out); nothing of it is in flight, and the rest is abandoned
          ok = false;
        } else if (ok) {
          const int64_t t = blockIdx.x + it * gridDim.x;
          const int b = (int)(t / H);
          const int h = (int)(t % H);
          const int hq = h / ratio;
          const bool rs_ok = rs_j >= 0 && rs_j < p.src_slots;
          const bool ws_ok = ws_j >= 0 && ws_j < p.dst_slots;
          bool mask_ok = true;
          if constexpr (C::kQ8) {
            // a head's masks must mark exactly n_hp rows, or the row ranks leave the tile
            int cs = 0, cd = 0;
#pragma unroll
            for (int w = 0; w < DK / 32; ++w) {
              cs += __popc(__ldg(p.src_mask + h * (DK / 32) + w));
              cd += __popc(__ldg(p.dst_mask + h * (DK / 32) + w));
            }
            mask_ok = cs == p.n_hp && cd == p.n_hp;
            if (!mask_ok) report(p.err, LA_DEVERR_Q8_MASK);
          }
          StepMeta m;
          m.g = g_j;
          m.beta = b_j;
          m.valid = rs_ok && ws_ok && mask_ok;
          m.ws = ws_j;
          m.dst_off = ((int64_t)ws_j * H + h) * tile_bytes;
          m.o_off = t * qg * DV;  // o row of the tile's first query
          meta[stage] = m;
          if (m.valid) {
            unsigned char* sb = smem + stage * C::kStageBytes;
            // query rows: the tile's q/k head, or its qg consecutive query heads
            const int64_t qrow = QGRP ? t * qg : (int64_t)b * p.n_qk_heads + hq;
            const int hist_bytes = CONV ? (2 * DK + DV) * (p.conv_w - 1) * (int)sizeof(IT) : 0;
            const int wbytes = CONV ? (2 * DK + DV) * p.conv_w * 4 : 0;
            mbar_arrive_expect_tx(&full[stage],
                                  C::kOffHist - C::kOffK + tile_bytes + qg * C::kQKBytes + hist_bytes + wbytes);
            bulk_g2s_hint(sb, src + ((int64_t)rs_j * H + h) * tile_bytes, tile_bytes, &full[stage], pol_stream);
            bulk_g2s(sb + C::kTileBytes, q + qrow * DK, qg * C::kQKBytes, &full[stage]);
            bulk_g2s(sb + C::kOffK, k + ((int64_t)b * p.n_qk_heads + hq) * DK, C::kQKBytes, &full[stage]);
            bulk_g2s(sb + C::kOffV, v + t * DV, C::kVBytes, &full[stage]);
            if (CHG) bulk_g2s(sb + C::kOffA, p.g + t * DK, C::kGBytes, &full[stage]);
            if (CONV) {
              bulk_g2s(sb + C::kOffHist,
                       static_cast<const unsigned char*>(p.conv_src) + ((int64_t)rs_j * H + h) * hist_bytes,
                       hist_bytes, &full[stage]);
              // the weights of the tile's q/k head and head (the same for every request)
              const int W = p.conv_w;
              bulk_g2s(sb + C::kOffConvW, p.conv_wq + (int64_t)hq * DK * W, DK * W * 4, &full[stage]);
              bulk_g2s(sb + C::kOffConvW + DK * W * 4, p.conv_wk + (int64_t)hq * DK * W, DK * W * 4, &full[stage]);
              bulk_g2s(sb + C::kOffConvW + 2 * DK * W * 4, p.conv_wv + (int64_t)h * DV * W, DV * W * 4,
                       &full[stage]);
            }
          } else {
            if (!rs_ok || !ws_ok) report(p.err, (rs_ok ? 0u : LA_DEVERR_READ_SLOT) | (ws_ok ? 0u : LA_DEVERR_WRITE_SLOT));
            mbar_arrive(&full[stage]);
          }
        } else {
          report(p.err, LA_DEVERR_TIMEOUT);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        abort = true;
        break;
      }
      ++issued;
    }
  }
  // Never retire with copies in flight: wait for the last phase issued on each stage.
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      if (issued > s) {
        const int64_t last = issued - 1 - ((issued - 1 - s) % C::kStages);
        if (blockIdx.x == 0 && last == p.withhold) continue;  // withheld: nothing issued
        if (!mbar_wait(&full[s], (uint32_t)(last / C::kStages) & 1u, p.wait_ns)) report(p.err, LA_DEVERR_TIMEOUT);
      }
    }
  }
}

// QGRP: the query-group direction of the ONNX operator -- k has one head per state head
// and p.q_group query heads (consecutive) read each state head; every extra query costs
// one more pass over the registers, the state is still read and written once.
template <int RULE, int DK, int DV, typename ST, typename IT, bool QGRP, bool CONV>
__global__ void __launch_bounds__(
    StepCfg<DK, DV, ST, IT, Rule<RULE>::kChannelGate, QGRP ? kMaxQueryGroup : 1, CONV>::kThreads, 1)
    step_kernel(const StepParams p) {
  constexpr bool CHG = Rule<RULE>::kChannelGate;
  using C = StepCfg<DK, DV, ST, IT, CHG, QGRP ? kMaxQueryGroup : 1, CONV>;
  static_assert(!(CONV && QGRP), "the convolution runs in the default head direction");
  const int qg = QGRP ? p.q_group : 1;
  extern __shared__ __align__(128) unsigned char smem[];
  StepMeta* meta = reinterpret_cast<StepMeta*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* empty = full + C::kStages;
  uint64_t* conv_done = empty + C::kStages;  // CONV

  const int H = p.n_v_heads;
  const int64_t ntiles = (int64_t)p.B * H;
  const int64_t n_my = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kWPT);
      if (CONV) mbar_init(&conv_done[s], C::kConvWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();
#if LA_STEP_PDL
  // Programmatic dependent launch: everything above overlapped the previous kernel on
  // the stream; nothing global is read before that kernel has completed.
  griddep_wait();
  griddep_launch_dependents();
#endif

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == C::kProducerWarp) {
    step_producer<RULE, DK, DV, ST, IT, QGRP, CONV, C>(p, smem, meta, full, empty, n_my, lane);
    return;
  }
  if constexpr (CONV) {
    if (warp >= C::kConsumerWarps) {
      conv_group<DK, DV, IT, C>(p, smem, meta, full, conv_done, n_my, warp - C::kConsumerWarps, lane);
      return;
    }
  }

  // -------------------------------------------------------------------- consumers
  constexpr int RL = C::kRL;
  constexpr int V = C::kVec;
  const int team = warp / C::kWPT;
  const int part = warp % C::kWPT;
  const int ch = lane % C::kNCH;              // 16-byte column chunk within the strip
  const int rb = lane / C::kNCH;              // row block
  const int col0 = part * C::kCW + ch * V;    // first column held by this lane
  const int row0 = rb * RL;                   // first row held by this lane
  unsigned char* dst = static_cast<unsigned char*>(p.dst);
  IT* out = static_cast<IT*>(p.o);
  // q8: INT8 rows of the source / destination tiles (BF16 rows follow the codes and scales)
  const int n8s = DK - p.n_hp, n8d = DK - p.n_hp;
  constexpr int NG = DV / 32;

  for (int64_t it = team; it < n_my; it += C::kTeams) {
    const int stage = (int)(it % C::kStages);
    const uint32_t round = (uint32_t)(it / C::kStages);
    bool arrived = mbar_wait(&full[stage], round & 1u, p.wait_ns);
    if (CONV && arrived) arrived = mbar_wait(&conv_done[stage], round & 1u, p.wait_ns);  // the tile's q, k, v
    const bool ok = __all_sync(0xffffffffu, arrived);
    if (!ok) {
      if (lane == 0) report(p.err, LA_DEVERR_TIMEOUT);
      return;
    }
    const StepMeta m = meta[stage];
    const unsigned char* sb = smem + stage * C::kStageBytes;
    // q, k, v of the step: the staged rows, or (CONV) the stage's post-convolution scratch
    using OT = std::conditional_t<CONV, float, IT>;
    const OT* qs;
    const OT* ks;
    const OT* vs;
    if constexpr (CONV) {
      const float* scr = reinterpret_cast<const float*>(smem + C::kOffScratch) + stage * C::kScrFloats;
      qs = scr;
      ks = scr + DK;
      vs = scr + 2 * DK;
    } else {
      qs = reinterpret_cast<const IT*>(sb + C::kTileBytes);
      ks = reinterpret_cast<const IT*>(sb + C::kOffK);
      vs = reinterpret_cast<const IT*>(sb + C::kOffV);
    }
    const float* as = reinterpret_cast<const float*>(sb + C::kOffA);
    float a, bcoef, c;
    Rule<RULE>::coeffs(m.g, m.beta, a, bcoef, c);

    float s[RL][V];
    Q8Rows<DK> rows_src, rows_dst;  // (q8) this lane's rows in the source / destination masks
    if constexpr (C::kQ8) {
      // q8 tile: this lane's rows from the INT8 codes (with their group's scale; the strip
      // is one 32-column group) or from the BF16 rows, as the head's mask says
      const int h = (int)((blockIdx.x + it * gridDim.x) % H);
      rows_src.init(p.src_mask + h * (DK / 32), row0);
      rows_dst.init(p.dst_mask + h * (DK / 32), row0);
#pragma unroll
      for (int r = 0; r < RL; ++r) {
        int idx;
        if (rows_src.row(r, idx)) {
          const uint4 w = *reinterpret_cast<const uint4*>(sb + n8s * DV + n8s * NG * 4 + (idx * DV + col0) * 2);
          StateVec<__nv_bfloat16>::unpack(w, s[r]);
        } else {
          const uint2 w = *reinterpret_cast<const uint2*>(sb + idx * DV + col0);
          const float sc = *reinterpret_cast<const float*>(sb + n8s * DV + (idx * NG + part) * 4);
          const uint32_t ww[2] = {w.x, w.y};
          q8_unpack<8>(ww, sc, s[r]);
        }
      }
    } else {
      const ST* tile = reinterpret_cast<const ST*>(sb);
#pragma unroll
      for (int r = 0; r < RL; ++r)
        StateVec<ST>::unpack(*reinterpret_cast<const uint4*>(tile + (row0 + r) * DV + col0), s[r]);
    }

    // k.q, S^T k and S^T q over this lane's rows (k, q read from the stage in blocks of
    // up to 8 rows), then across the row blocks.  kda: the rows' decays scale the keys of
    // both sums, (Diag(alpha) S)^T k and (Diag(alpha) S)^T q; k.q stays undecayed.
    constexpr int KB = RL < 8 ? RL : 8;
    float kq = 0.0f;
    float2 pp[V / 2], rr[V / 2];
#pragma unroll
    for (int j = 0; j < V / 2; ++j) pp[j] = rr[j] = f2(0.0f, 0.0f);
#pragma unroll
    for (int r0 = 0; r0 < RL; r0 += KB) {
      float kb[KB], qb[KB], ab[KB];
      load_f32<OT, KB>(ks + row0 + r0, kb);
      load_f32<OT, KB>(qs + row0 + r0, qb);
      if (CHG) load_f32<float, KB>(as + row0 + r0, ab);
#pragma unroll
      for (int r = 0; r < KB; ++r) {
        kq = fmaf(kb[r], qb[r], kq);
        const float kr = CHG ? kb[r] * ab[r] : kb[r];
        const float qr = CHG ? qb[r] * ab[r] : qb[r];
        const float2 k2 = f2(kr, kr);
        const float2 q2 = f2(qr, qr);
#pragma unroll
        for (int j = 0; j < V / 2; ++j) {
          const float2 s2 = f2(s[r0 + r][2 * j], s[r0 + r][2 * j + 1]);
          if (Rule<RULE>::kPredicts) pp[j] = fma2(s2, k2, pp[j]);
          rr[j] = fma2(s2, q2, rr[j]);
        }
      }
    }
#pragma unroll
    for (int off = C::kNCH; off < 32; off <<= 1) {
      kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
      for (int j = 0; j < V / 2; ++j) {
        if (Rule<RULE>::kPredicts) {
          pp[j].x += __shfl_xor_sync(0xffffffffu, pp[j].x, off);
          pp[j].y += __shfl_xor_sync(0xffffffffu, pp[j].y, off);
        }
        rr[j].x += __shfl_xor_sync(0xffffffffu, rr[j].x, off);
        rr[j].y += __shfl_xor_sync(0xffffffffu, rr[j].y, off);
      }
    }

    if (m.valid) {
      // u = b (v - c p),  o = scale (a r + (k.q) u)
      float vv[V], u[V], o[V];
      load_f32<OT, V>(vs + col0, vv);
#pragma unroll
      for (int j = 0; j < V / 2; ++j) {
        u[2 * j] = bcoef * (vv[2 * j] - c * pp[j].x);
        u[2 * j + 1] = bcoef * (vv[2 * j + 1] - c * pp[j].y);
        o[2 * j] = p.scale * fmaf(a, rr[j].x, kq * u[2 * j]);
        o[2 * j + 1] = p.scale * fmaf(a, rr[j].y, kq * u[2 * j + 1]);
      }
      if (rb == 0) store_f32<IT, V>(out + m.o_off + col0, o);

      // the group's other queries read the same updated state: o = scale (a S^T q + (k.q) u)
      if (QGRP) {
#pragma unroll 1
        for (int qi = 1; qi < qg; ++qi) {
          float kqi = 0.0f;
          float2 ri[V / 2];
#pragma unroll
          for (int j = 0; j < V / 2; ++j) ri[j] = f2(0.0f, 0.0f);
#pragma unroll
          for (int r0 = 0; r0 < RL; r0 += KB) {
            float kb[KB], qb[KB], ab[KB];
            load_f32<OT, KB>(ks + row0 + r0, kb);
            load_f32<OT, KB>(qs + qi * DK + row0 + r0, qb);
            if (CHG) load_f32<float, KB>(as + row0 + r0, ab);
#pragma unroll
            for (int r = 0; r < KB; ++r) {
              kqi = fmaf(kb[r], qb[r], kqi);
              const float qr = CHG ? qb[r] * ab[r] : qb[r];
              const float2 q2 = f2(qr, qr);
#pragma unroll
              for (int j = 0; j < V / 2; ++j) ri[j] = fma2(f2(s[r0 + r][2 * j], s[r0 + r][2 * j + 1]), q2, ri[j]);
            }
          }
#pragma unroll
          for (int off = C::kNCH; off < 32; off <<= 1) {
            kqi += __shfl_xor_sync(0xffffffffu, kqi, off);
#pragma unroll
            for (int j = 0; j < V / 2; ++j) {
              ri[j].x += __shfl_xor_sync(0xffffffffu, ri[j].x, off);
              ri[j].y += __shfl_xor_sync(0xffffffffu, ri[j].y, off);
            }
          }
#pragma unroll
          for (int j = 0; j < V / 2; ++j) {
            o[2 * j] = p.scale * fmaf(a, ri[j].x, kqi * u[2 * j]);
            o[2 * j + 1] = p.scale * fmaf(a, ri[j].y, kqi * u[2 * j + 1]);
          }
          if (rb == 0) store_f32<IT, V>(out + m.o_off + qi * DV + col0, o);
        }
      }

      // S' = a S + k u^T, stored with 16-byte vectors (q8: 8 codes or 8 BF16 values)
      unsigned char* dtile = dst + m.dst_off;
      const float2 a2 = f2(a, a);
#pragma unroll
      for (int r0 = 0; r0 < RL; r0 += KB) {
        float kb[KB], ab[KB];
        load_f32<OT, KB>(ks + row0 + r0, kb);
        if (CHG) load_f32<float, KB>(as + row0 + r0, ab);
#pragma unroll
        for (int r = 0; r < KB; ++r) {
          const float2 k2 = f2(kb[r], kb[r]);
          const float2 ar = CHG ? f2(ab[r], ab[r]) : a2;
          float y[V];
#pragma unroll
          for (int j = 0; j < V / 2; ++j) {
            const float2 t =
                fma2(k2, f2(u[2 * j], u[2 * j + 1]), mul2(ar, f2(s[r0 + r][2 * j], s[r0 + r][2 * j + 1])));
            y[2 * j] = t.x;
            y[2 * j + 1] = t.y;
          }
          if constexpr (C::kQ8) {
            // group absmax over the 4 lanes holding this row of the strip
            float amax = 0.0f;
#pragma unroll
            for (int e = 0; e < V; ++e) amax = fmaxf(amax, fabsf(y[e]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            int idx;
            if (rows_dst.row(r0 + r, idx)) {
              *reinterpret_cast<uint4*>(dtile + n8d * DV + n8d * NG * 4 + (idx * DV + col0) * 2) =
                  StateVec<__nv_bfloat16>::pack(y);
            } else {
              float sc, inv;
              q8_scales(amax, sc, inv);
              uint32_t w[2];
              q8_pack<8>(y, inv, w);
              *reinterpret_cast<uint2*>(dtile + idx * DV + col0) = make_uint2(w[0], w[1]);
              if (ch == 0) *reinterpret_cast<float*>(dtile + n8d * DV + (idx * NG + part) * 4) = sc;
            }
          } else {
            *reinterpret_cast<uint4*>(reinterpret_cast<ST*>(dtile) + (row0 + r0 + r) * DV + col0) =
                StateVec<ST>::pack(y);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
  }
}

template <int RULE, int DK, int DV, typename ST, typename IT, bool QGRP, bool CONV = false>
cudaError_t launch_step(const StepParams& p, cudaStream_t stream) {
  using C = StepCfg<DK, DV, ST, IT, Rule<RULE>::kChannelGate, QGRP ? kMaxQueryGroup : 1, CONV>;
  const void* fn = reinterpret_cast<const void*>(&step_kernel<RULE, DK, DV, ST, IT, QGRP, CONV>);
  const int per_sm = prepare_kernel(fn, C::kThreads, C::kSmem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  const int64_t ntiles = (int64_t)p.B * p.n_v_heads;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)(ntiles < cap ? ntiles : cap);
#if LA_STEP_PDL
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, step_kernel<RULE, DK, DV, ST, IT, QGRP, CONV>, p);
  if (e != cudaSuccess) return e;
#else
  step_kernel<RULE, DK, DV, ST, IT, QGRP, CONV><<<grid, C::kThreads, C::kSmem, stream>>>(p);
#endif
  return cudaGetLastError();
}

// Launcher table for one state dtype and head direction: rule x (d_k, d_v) x io dtype.
template <typename ST, bool QGRP>
StepLaunchFn find_step_impl(int rule, int dk, int dv, int io) {
#define LA_STEP_CASE(R, K, V)                                                                    \
  if (rule == R && dk == K && dv == V)                                                           \
    return io == LA_F32 ? &launch_step<R, K, V, ST, float, QGRP> : &launch_step<R, K, V, ST, __nv_bfloat16, QGRP>;
#define LA_STEP_SHAPES(R) LA_STEP_CASE(R, 16, 16) LA_STEP_CASE(R, 64, 64) LA_STEP_CASE(R, 128, 64) LA_STEP_CASE(R, 128, 128)
  LA_STEP_SHAPES(LA_RULE_LINEAR)
  LA_STEP_SHAPES(LA_RULE_GATED)
  LA_STEP_SHAPES(LA_RULE_DELTA)
  LA_STEP_SHAPES(LA_RULE_GATED_DELTA)
  LA_STEP_SHAPES(LA_RULE_KDA)
#undef LA_STEP_SHAPES
#undef LA_STEP_CASE
  return nullptr;
}

// Launcher table of the q8 state storage (d_v a multiple of the 32-column group).
template <bool QGRP>
StepLaunchFn find_step_q8_impl(int rule, int dk, int dv, int io) {
#define LA_Q8_CASE(R, K, V)                                                                      \
  if (rule == R && dk == K && dv == V)                                                           \
    return io == LA_F32 ? &launch_step<R, K, V, q8_t, float, QGRP> : &launch_step<R, K, V, q8_t, __nv_bfloat16, QGRP>;
#define LA_Q8_SHAPES(R) LA_Q8_CASE(R, 64, 64) LA_Q8_CASE(R, 128, 64) LA_Q8_CASE(R, 128, 128)
  LA_Q8_SHAPES(LA_RULE_LINEAR)
  LA_Q8_SHAPES(LA_RULE_GATED)
  LA_Q8_SHAPES(LA_RULE_DELTA)
  LA_Q8_SHAPES(LA_RULE_GATED_DELTA)
  LA_Q8_SHAPES(LA_RULE_KDA)
#undef LA_Q8_SHAPES
#undef LA_Q8_CASE
  return nullptr;
}

// Launcher table of the step with the convolution fused ahead (FP32 or BF16 state).
template <typename ST>
StepLaunchFn find_step_conv_impl(int rule, int dk, int dv, int io) {
#define LA_CONV_CASE(R, K, V)                                                                    \
  if (rule == R && dk == K && dv == V)                                                           \
    return io == LA_F32 ? &launch_step<R, K, V, ST, float, false, true>                          \
                        : &launch_step<R, K, V, ST, __nv_bfloat16, false, true>;
#define LA_CONV_SHAPES(R) LA_CONV_CASE(R, 16, 16) LA_CONV_CASE(R, 64, 64) LA_CONV_CASE(R, 128, 64) LA_CONV_CASE(R, 128, 128)
  LA_CONV_SHAPES(LA_RULE_LINEAR)
  LA_CONV_SHAPES(LA_RULE_GATED)
  LA_CONV_SHAPES(LA_RULE_DELTA)
  LA_CONV_SHAPES(LA_RULE_GATED_DELTA)
  LA_CONV_SHAPES(LA_RULE_KDA)
#undef LA_CONV_SHAPES
#undef LA_CONV_CASE
  return nullptr;
}

}  // namespace la
