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
//    "asynchronous state transfers" of the "Gated DeltaNet" page (How to read it) --
//    so that several tiles are in flight per SM at all times;
//  * every column of S evolves on its own, so each consumer warp owns a strip of up to
//    32 columns of a tile for all d_k rows and needs nobody else: lanes split the strip
//    into 16-byte column chunks x row blocks, hold the strip's 128 state values in FP32
//    registers, finish S^T k and S^T q with xor-shuffles inside the warp, form u and o,
//    release the stage on their own, and store the new state with 16-byte stores.
//    Warps of different tiles run concurrently; there is no CTA-wide barrier.  Four
//    consumer warps (plus the producer) keep every SM sub-partition at <= 2 warps so a
//    thread may hold its 128 state values without spilling.
//  * FP32 arithmetic in packed pairs (sm_100 FFMA2 / FMUL2).
#pragma once

#include <cstdint>

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
  int32_t pad;
  int64_t dst_off;  // element offset of the destination tile in the destination pool
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

template <int DK, int DV, typename ST, typename IT>
struct StepCfg {
  static constexpr int kSB = sizeof(ST);
  static constexpr int kVec = StateVec<ST>::kElems;     // state elements per 16-byte chunk
  static constexpr int kCW = DV < LA_STEP_STRIP_COLS ? DV : LA_STEP_STRIP_COLS;  // strip width
  static constexpr int kWPT = DV / kCW;                 // warps per tile
  static constexpr int kNCH = kCW / kVec;               // 16-byte chunks per strip row
  static constexpr int kRG = 32 / kNCH;                 // row blocks per warp
  static constexpr int kRL = DK / kRG;                  // rows per lane
  static constexpr int kConsumerWarps = kWPT > LA_STEP_CONSUMER_WARPS ? kWPT : LA_STEP_CONSUMER_WARPS;
  static constexpr int kTeams = kConsumerWarps / kWPT;  // tiles in compute at once
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  static constexpr int kTileBytes = DK * DV * kSB;
  static constexpr int kQKBytes = DK * (int)sizeof(IT);
  static constexpr int kVBytes = DV * (int)sizeof(IT);
  static constexpr int kCopyBytes = kTileBytes + 2 * kQKBytes + kVBytes;
  static constexpr int kStageBytes = round_up(kCopyBytes, 128);
  static constexpr int kStages = cmax(2, cmin(12, (204 * 1024) / kStageBytes));
  static constexpr int kOffMeta = kStages * kStageBytes;
  static constexpr int kOffBars = round_up(kOffMeta + kStages * (int)sizeof(StepMeta), 8);
  static constexpr int kSmem = kOffBars + 2 * kStages * 8;

  static_assert(kNCH >= 1 && kNCH <= 32 && (32 % kNCH) == 0, "strip row must map onto a power-of-two lane group");
  static_assert(kRL >= 1 && DK % kRG == 0, "rows must split evenly over the row blocks");
  static_assert(kConsumerWarps % kWPT == 0, "whole tiles per team");
  static_assert(kQKBytes % 16 == 0 && kVBytes % 16 == 0 && kTileBytes % 16 == 0, "bulk copies move 16-byte units");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int RULE, int DK, int DV, typename ST, typename IT>
__global__ void __launch_bounds__(StepCfg<DK, DV, ST, IT>::kThreads, 1) step_kernel(const StepParams p) {
  using C = StepCfg<DK, DV, ST, IT>;
  extern __shared__ __align__(128) unsigned char smem[];
  StepMeta* meta = reinterpret_cast<StepMeta*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* empty = full + C::kStages;

  const int H = p.n_v_heads;
  const int64_t ntiles = (int64_t)p.B * H;
  const int64_t n_my = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kWPT);
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

  if (warp == C::kConsumerWarps) {
    // ------------------------------------------------------------------ producer
    const uint64_t pol_stream = policy_evict_first();
    const int ratio = H / p.n_qk_heads;
    const ST* src = static_cast<const ST*>(p.src);
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
          ok = mbar_wait(&empty[stage], (round & 1u) ^ 1u);
          if (ok) {
            const int64_t t = blockIdx.x + it * gridDim.x;
            const int b = (int)(t / H);
            const int h = (int)(t % H);
            const int hq = h / ratio;
            const bool rs_ok = rs_j >= 0 && rs_j < p.src_slots;
            const bool ws_ok = ws_j >= 0 && ws_j < p.dst_slots;
            StepMeta m;
            m.g = g_j;
            m.beta = b_j;
            m.valid = rs_ok && ws_ok;
            m.pad = 0;
            m.dst_off = ((int64_t)ws_j * H + h) * (DK * DV);
            m.o_off = t * DV;
            meta[stage] = m;
            if (m.valid) {
              unsigned char* sb = smem + stage * C::kStageBytes;
              mbar_arrive_expect_tx(&full[stage], C::kCopyBytes);
              bulk_g2s_hint(sb, src + ((int64_t)rs_j * H + h) * (DK * DV), C::kTileBytes, &full[stage], pol_stream);
              bulk_g2s(sb + C::kTileBytes, q + ((int64_t)b * p.n_qk_heads + hq) * DK, C::kQKBytes, &full[stage]);
              bulk_g2s(sb + C::kTileBytes + C::kQKBytes, k + ((int64_t)b * p.n_qk_heads + hq) * DK, C::kQKBytes,
                       &full[stage]);
              bulk_g2s(sb + C::kTileBytes + 2 * C::kQKBytes, v + t * DV, C::kVBytes, &full[stage]);
            } else {
              report(p.err, (rs_ok ? 0u : LA_DEVERR_READ_SLOT) | (ws_ok ? 0u : LA_DEVERR_WRITE_SLOT));
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
          if (!mbar_wait(&full[s], (uint32_t)(last / C::kStages) & 1u)) report(p.err, LA_DEVERR_TIMEOUT);
        }
      }
    }
    return;
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
  ST* dst = static_cast<ST*>(p.dst);
  IT* out = static_cast<IT*>(p.o);

  for (int64_t it = team; it < n_my; it += C::kTeams) {
    const int stage = (int)(it % C::kStages);
    const uint32_t round = (uint32_t)(it / C::kStages);
    const bool arrived = mbar_wait(&full[stage], round & 1u);
    if (!__all_sync(0xffffffffu, arrived)) {
      if (lane == 0) report(p.err, LA_DEVERR_TIMEOUT);
      return;
    }
    const StepMeta m = meta[stage];
    const unsigned char* sb = smem + stage * C::kStageBytes;
    const ST* tile = reinterpret_cast<const ST*>(sb);
    const IT* qs = reinterpret_cast<const IT*>(sb + C::kTileBytes);
    const IT* ks = reinterpret_cast<const IT*>(sb + C::kTileBytes + C::kQKBytes);
    const IT* vs = reinterpret_cast<const IT*>(sb + C::kTileBytes + 2 * C::kQKBytes);
    float a, bcoef, c;
    Rule<RULE>::coeffs(m.g, m.beta, a, bcoef, c);

    float s[RL][V];
#pragma unroll
    for (int r = 0; r < RL; ++r)
      StateVec<ST>::unpack(*reinterpret_cast<const uint4*>(tile + (row0 + r) * DV + col0), s[r]);

    // k.q, S^T k and S^T q over this lane's rows (k, q read from the stage in blocks of
    // up to 8 rows), then across the row blocks
    constexpr int KB = RL < 8 ? RL : 8;
    float kq = 0.0f;
    float2 pp[V / 2], rr[V / 2];
#pragma unroll
    for (int j = 0; j < V / 2; ++j) pp[j] = rr[j] = f2(0.0f, 0.0f);
#pragma unroll
    for (int r0 = 0; r0 < RL; r0 += KB) {
      float kb[KB], qb[KB];
      load_f32<IT, KB>(ks + row0 + r0, kb);
      load_f32<IT, KB>(qs + row0 + r0, qb);
#pragma unroll
      for (int r = 0; r < KB; ++r) {
        kq = fmaf(kb[r], qb[r], kq);
        const float2 k2 = f2(kb[r], kb[r]);
        const float2 q2 = f2(qb[r], qb[r]);
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
      load_f32<IT, V>(vs + col0, vv);
#pragma unroll
      for (int j = 0; j < V / 2; ++j) {
        u[2 * j] = bcoef * (vv[2 * j] - c * pp[j].x);
        u[2 * j + 1] = bcoef * (vv[2 * j + 1] - c * pp[j].y);
        o[2 * j] = p.scale * fmaf(a, rr[j].x, kq * u[2 * j]);
        o[2 * j + 1] = p.scale * fmaf(a, rr[j].y, kq * u[2 * j + 1]);
      }
      if (rb == 0) store_f32<IT, V>(out + m.o_off + col0, o);

      // S' = a S + k u^T, stored with 16-byte vectors
      ST* dtile = dst + m.dst_off;
      const float2 a2 = f2(a, a);
#pragma unroll
      for (int r0 = 0; r0 < RL; r0 += KB) {
        float kb[KB];
        load_f32<IT, KB>(ks + row0 + r0, kb);
#pragma unroll
        for (int r = 0; r < KB; ++r) {
          const float2 k2 = f2(kb[r], kb[r]);
          float y[V];
#pragma unroll
          for (int j = 0; j < V / 2; ++j) {
            const float2 t =
                fma2(k2, f2(u[2 * j], u[2 * j + 1]), mul2(a2, f2(s[r0 + r][2 * j], s[r0 + r][2 * j + 1])));
            y[2 * j] = t.x;
            y[2 * j + 1] = t.y;
          }
          *reinterpret_cast<uint4*>(dtile + (row0 + r0 + r) * DV + col0) = StateVec<ST>::pack(y);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
  }
}

template <int RULE, int DK, int DV, typename ST, typename IT>
cudaError_t launch_step(const StepParams& p, cudaStream_t stream) {
  using C = StepCfg<DK, DV, ST, IT>;
  const void* fn = reinterpret_cast<const void*>(&step_kernel<RULE, DK, DV, ST, IT>);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, step_kernel<RULE, DK, DV, ST, IT>, p);
  if (e != cudaSuccess) return e;
#else
  step_kernel<RULE, DK, DV, ST, IT><<<grid, C::kThreads, C::kSmem, stream>>>(p);
#endif
  return cudaGetLastError();
}

// Launcher table for one state dtype: rule x (d_k, d_v) x io dtype.
template <typename ST>
StepLaunchFn find_step_impl(int rule, int dk, int dv, int io) {
#define LA_STEP_CASE(R, K, V)                                                                    \
  if (rule == R && dk == K && dv == V)                                                           \
    return io == LA_F32 ? &launch_step<R, K, V, ST, float> : &launch_step<R, K, V, ST, __nv_bfloat16>;
#define LA_STEP_SHAPES(R) LA_STEP_CASE(R, 16, 16) LA_STEP_CASE(R, 64, 64) LA_STEP_CASE(R, 128, 64) LA_STEP_CASE(R, 128, 128)
  LA_STEP_SHAPES(LA_RULE_LINEAR)
  LA_STEP_SHAPES(LA_RULE_GATED)
  LA_STEP_SHAPES(LA_RULE_DELTA)
  LA_STEP_SHAPES(LA_RULE_GATED_DELTA)
#undef LA_STEP_SHAPES
#undef LA_STEP_CASE
  return nullptr;
}

}  // namespace la
