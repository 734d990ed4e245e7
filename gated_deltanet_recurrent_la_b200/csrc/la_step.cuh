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
//    with 1-D bulk copies on the TMA engine, signalling an mbarrier; the "asynchronous
//    state transfers" of the "Gated DeltaNet" page (How to read it), so several tiles
//    are always in flight per SM;
//  * eight consumer warps turn a stage into FP32 registers (16-byte vectors, 8 BF16 or
//    4 FP32 state elements per thread per row), reduce S^T k and S^T q over d_k with
//    shuffles plus one shared-memory pass, form u and o, release the stage, and store
//    the new state with coalesced 16-byte stores (BF16 rounding to nearest even).
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

template <int DK, int DV, typename ST, typename IT>
struct StepCfg {
  static constexpr int kSB = sizeof(ST);
  static constexpr int kVec = StateVec<ST>::kElems;  // state elements per 16-byte vector
  static constexpr int kTPR = DV / kVec;             // threads covering one row of the tile
  static constexpr int kConsumerWarps = 8;
  static constexpr int kConsumers = kConsumerWarps * 32;
  static constexpr int kThreads = kConsumers + 32;   // + one producer warp
  static constexpr int kUsed = cmin(DK * kTPR, kConsumers);  // consumer threads holding state
  static constexpr int kUsedWarps = kUsed / 32;
  static constexpr int kRowsPerPass = kUsed / kTPR;
  static constexpr int kPasses = DK / kRowsPerPass;  // rows per thread
  static constexpr int kTileBytes = DK * DV * kSB;
  static constexpr int kQKBytes = DK * (int)sizeof(IT);
  static constexpr int kVBytes = DV * (int)sizeof(IT);
  static constexpr int kCopyBytes = kTileBytes + 2 * kQKBytes + kVBytes;
  static constexpr int kStageBytes = round_up(kCopyBytes, 128);
  static constexpr int kStages = cmax(2, cmin(8, (200 * 1024) / kStageBytes));
  // shared-memory layout
  static constexpr int kOffMeta = kStages * kStageBytes;
  static constexpr int kOffRedP = round_up(kOffMeta + kStages * (int)sizeof(StepMeta), 16);
  static constexpr int kOffRedR = kOffRedP + kUsedWarps * DV * 4;
  static constexpr int kOffU = kOffRedR + kUsedWarps * DV * 4;
  static constexpr int kOffBars = round_up(kOffU + DV * 4, 8);
  static constexpr int kSmem = kOffBars + 2 * kStages * 8;

  static_assert(kTPR >= 1 && kTPR <= 32 && (32 % kTPR) == 0, "row must map onto a power-of-two lane group");
  static_assert(kUsed % 32 == 0 && DK % kRowsPerPass == 0, "tile must map onto whole warps");
  static_assert(kVec % 4 == 0 || kVec == 4, "vector width");
  static_assert(DV <= kConsumers, "one finishing thread per column");
  static_assert(kQKBytes % 16 == 0 && kVBytes % 16 == 0 && kTileBytes % 16 == 0, "bulk copies move 16-byte units");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int RULE, int DK, int DV, typename ST, typename IT>
__global__ void __launch_bounds__(StepCfg<DK, DV, ST, IT>::kThreads, 1) step_kernel(const StepParams p) {
  using C = StepCfg<DK, DV, ST, IT>;
  extern __shared__ __align__(128) unsigned char smem[];
  StepMeta* meta = reinterpret_cast<StepMeta*>(smem + C::kOffMeta);
  float* red_p = reinterpret_cast<float*>(smem + C::kOffRedP);
  float* red_r = reinterpret_cast<float*>(smem + C::kOffRedR);
  float* ubuf = reinterpret_cast<float*>(smem + C::kOffU);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* empty = full + C::kStages;

  const int H = p.n_v_heads;
  const int64_t ntiles = (int64_t)p.B * H;
  const int64_t n_my = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init_fence();
  }
  __syncthreads();

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
  const int tid = threadIdx.x;  // 0 .. kConsumers-1
  const bool holds = tid < C::kUsed;
  const int cc = tid % C::kTPR;  // 16-byte column chunk
  const int r0 = tid / C::kTPR;  // first row
  ST* dst = static_cast<ST*>(p.dst);
  IT* out = static_cast<IT*>(p.o);

  for (int64_t it = 0; it < n_my; ++it) {
    const int stage = (int)(it % C::kStages);
    const uint32_t round = (uint32_t)(it / C::kStages);
    const bool arrived = mbar_wait(&full[stage], round & 1u);
    const StepMeta m = meta[stage];
    const unsigned char* sb = smem + stage * C::kStageBytes;
    const ST* tile = reinterpret_cast<const ST*>(sb);
    const IT* qs = reinterpret_cast<const IT*>(sb + C::kTileBytes);
    const IT* ks = reinterpret_cast<const IT*>(sb + C::kTileBytes + C::kQKBytes);
    const IT* vs = reinterpret_cast<const IT*>(sb + C::kTileBytes + 2 * C::kQKBytes);
    float a, bcoef, c;
    Rule<RULE>::coeffs(m.g, m.beta, a, bcoef, c);

    // k . q (every warp computes it; only the finishing threads use it)
    float kq = 0.0f;
    for (int i = lane; i < DK; i += 32) kq = fmaf(io_load(ks + i), io_load(qs + i), kq);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);

    float s[C::kPasses][C::kVec];
    float kr[C::kPasses];
    if (holds) {
      float pp[C::kVec], rr[C::kVec];
#pragma unroll
      for (int e = 0; e < C::kVec; ++e) pp[e] = rr[e] = 0.0f;
#pragma unroll
      for (int ps = 0; ps < C::kPasses; ++ps) {
        const int row = r0 + ps * C::kRowsPerPass;
        const uint4 w = *reinterpret_cast<const uint4*>(tile + row * DV + cc * C::kVec);
        StateVec<ST>::unpack(w, s[ps]);
        kr[ps] = io_load(ks + row);
        const float qr = io_load(qs + row);
#pragma unroll
        for (int e = 0; e < C::kVec; ++e) {
          if (Rule<RULE>::kPredicts) pp[e] = fmaf(s[ps][e], kr[ps], pp[e]);
          rr[e] = fmaf(s[ps][e], qr, rr[e]);
        }
      }
#pragma unroll
      for (int off = C::kTPR; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < C::kVec; ++e) {
          if (Rule<RULE>::kPredicts) pp[e] += __shfl_xor_sync(0xffffffffu, pp[e], off);
          rr[e] += __shfl_xor_sync(0xffffffffu, rr[e], off);
        }
      }
      if (lane < C::kTPR) {
        float4* dp = reinterpret_cast<float4*>(red_p + warp * DV + cc * C::kVec);
        float4* dr = reinterpret_cast<float4*>(red_r + warp * DV + cc * C::kVec);
#pragma unroll
        for (int e4 = 0; e4 < C::kVec / 4; ++e4) {
          if (Rule<RULE>::kPredicts) dp[e4] = make_float4(pp[4 * e4], pp[4 * e4 + 1], pp[4 * e4 + 2], pp[4 * e4 + 3]);
          dr[e4] = make_float4(rr[4 * e4], rr[4 * e4 + 1], rr[4 * e4 + 2], rr[4 * e4 + 3]);
        }
      }
    }
    // Barrier 1 (consumers): partial sums are in shared memory.  It also ORs the
    // "stage never arrived" flags so that every consumer leaves together.
    if (named_bar_or(1, C::kConsumers, !arrived)) {
      if (tid == 0) report(p.err, LA_DEVERR_TIMEOUT);
      return;
    }
    if (tid < DV) {
      float pj = 0.0f, rj = 0.0f;
#pragma unroll
      for (int w = 0; w < C::kUsedWarps; ++w) {
        if (Rule<RULE>::kPredicts) pj += red_p[w * DV + tid];
        rj += red_r[w * DV + tid];
      }
      const float u = bcoef * (io_load(vs + tid) - c * pj);
      ubuf[tid] = u;
      if (m.valid) io_store(out + m.o_off + tid, p.scale * fmaf(a, rj, kq * u));
    }
    // Barrier 2: u is in shared memory and nobody reads the stage any more.
    named_bar_sync(2, C::kConsumers);
    if (tid == 0) mbar_arrive(&empty[stage]);
    if (holds && m.valid) {
      float u[C::kVec];
#pragma unroll
      for (int e4 = 0; e4 < C::kVec / 4; ++e4) {
        const float4 x = *reinterpret_cast<const float4*>(ubuf + cc * C::kVec + 4 * e4);
        u[4 * e4] = x.x; u[4 * e4 + 1] = x.y; u[4 * e4 + 2] = x.z; u[4 * e4 + 3] = x.w;
      }
      ST* dtile = dst + m.dst_off;
#pragma unroll
      for (int ps = 0; ps < C::kPasses; ++ps) {
        const int row = r0 + ps * C::kRowsPerPass;
        float y[C::kVec];
#pragma unroll
        for (int e = 0; e < C::kVec; ++e) y[e] = fmaf(kr[ps], u[e], a * s[ps][e]);
        *reinterpret_cast<uint4*>(dtile + row * DV + cc * C::kVec) = StateVec<ST>::pack(y);
      }
    }
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
  step_kernel<RULE, DK, DV, ST, IT><<<grid, C::kThreads, C::kSmem, stream>>>(p);
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
