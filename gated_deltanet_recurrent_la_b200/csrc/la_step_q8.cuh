// la_step_q8.cuh -- the decode step on q8 state pools whose source and destination share
// one channel mask (the in-place decode of a serving pool: the same pool, or pools with
// the same mask array).
//
// The q8 format (DAMP-style mixed storage, "Seven Architectures Replacing KV Cache With
// Bounded Mutable State", sections "ONNX LinearAttention / FlashInfer" and Practical
// Implications) stores a tile's rows in two blocks: the INT8 rows (codes, then one FP32
// scale per 32 columns) and the BF16 rows, each block in increasing key channel.  With one
// mask for both tiles a row has the same place in the source and the destination, so the
// lanes here walk the rows in that storage order.  Each warp owns one 32-column group (a
// strip) of a tile; lane (rb, hf) holds columns hf * 16 .. hf * 16 + 15 of the strip in the
// storage rows 16 m + rb (m = 0 .. d_k / 16 - 1), the INT8 rows first.  At each m all lanes
// then see the same kind of row (when the number of INT8 rows is a multiple of 16;
// otherwise one m is mixed), so the warp does not diverge, and the key channel of a row
// only matters for its key, query and decay, which each warp gathers once per tile into
// row order.  A group's absmax is one shuffle between the two halves, and its scale is
// computed once per 16 values.
//
// Arithmetic (same update and readout as the other step kernels, FP32):
//  * an INT8 row is held as its exact integer codes and the group scale s; the sums take
//    sum_i code_ij (s_i k_i), the update a S + k u^T takes code (a s) + k u;
//  * codes become floats without the conversion unit: the byte, offset by 128, placed in
//    the mantissa of 2^23 and 2^23 + 128 subtracted (exact);
//  * new codes are rint(y * inv) as the codec rounds them: the product rounded to FP32, then
//    added to 1.5 * 2^23, whose low byte is then the two's-complement code (exact for
//    |y * inv| < 2^22, and |y * inv| <= 127.00002 here);  a row group holding a non-finite
//    value (rare) takes the codec's own conversion, which sends NaN to 0;
//  * the pairwise products run as packed FP32 pairs (FFMA2 / FMUL2 / FADD2: the same
//    correctly rounded results as two scalar operations, half the instructions);
//  * the column sums S^T k and S^T q meet across the 16 row blocks by recursive halving
//    (each lane ends with the two sums of one column, which gives that column's u and o);
//    u goes to the warp's lanes through shared memory;
//  * two passes over the staged tile (sums, then update and store) instead of holding the
//    tile in registers: a thread needs few registers (at most 96 with 17 warps), so four
//    tiles are in compute per SM (sixteen consumer warps) to hide the latencies of one warp
//    per tile strip.
#pragma once

#include "la_step.cuh"

namespace la {

#ifndef LA_Q8S_CONSUMER_WARPS
#define LA_Q8S_CONSUMER_WARPS 16
#endif

// Stage layout of the generic step (StepCfg) with NCW consumer warps, each with its own
// row-ordered key / query / decay vectors and a u vector of its strip after the stages.
template <int DK, int DV, typename IT, bool CHG, int NCW>
struct Q8sCfg : StepCfg<DK, DV, q8_t, IT, CHG> {
  using Base = StepCfg<DK, DV, q8_t, IT, CHG>;
  static constexpr int kConsumerWarps = NCW;
  static constexpr int kTeams = NCW / Base::kWPT;
  static constexpr int kThreads = (NCW + 1) * 32;
  static constexpr int kPermFloats = 3 * DK + 32;  // k | q | alpha (lane-major row order) | u
  static constexpr int kFixed = NCW * kPermFloats * 4 + 12 * ((int)sizeof(StepMeta) + 16) + 64;
  static constexpr int kStages = cmax(2, cmin(12, (227 * 1024 - kFixed) / Base::kStageBytes));
  static constexpr int kOffMeta = kStages * Base::kStageBytes;
  static constexpr int kOffBars = round_up(kOffMeta + kStages * (int)sizeof(StepMeta), 8);
  static constexpr int kOffPerm = round_up(kOffBars + 2 * kStages * 8, 16);
  static constexpr int kSmem = kOffPerm + NCW * kPermFloats * 4;
  static_assert(NCW % Base::kWPT == 0, "whole tiles per team");
  static_assert(DV % 32 == 0 && DK % 64 == 0, "32-column strips, 16 row blocks of a multiple of 4 rows");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// max that keeps a NaN (so that one compare tells a row group holding a non-finite value)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// N signed codes (little-endian bytes of N / 4 words) -> their exact values as floats
template <int N>
__device__ __forceinline__ void q8s_codes(const uint32_t* words, float* c) {
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const uint32_t x = words[i] ^ 0x80808080u;
#pragma unroll
    for (int b = 0; b < 4; ++b) c[4 * i + b] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | b));
  }
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const float2 r = __fadd2_rn(make_float2(c[e], c[e + 1]), make_float2(-8388736.0f, -8388736.0f));
    c[e] = r.x;
    c[e + 1] = r.y;
  }
}

// codes rint(y * inv) of N finite values with |y| <= the group's absmax, packed into N bytes
template <int N>
__device__ __forceinline__ void q8s_pack(const float* y, float inv, uint32_t* w) {
  uint32_t b[N];
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const float2 r = __fadd2_rn(__fmul2_rn(make_float2(y[e], y[e + 1]), make_float2(inv, inv)),
                                make_float2(12582912.0f, 12582912.0f));
    b[e] = __float_as_uint(r.x);
    b[e + 1] = __float_as_uint(r.y);
  }
#pragma unroll
  for (int i = 0; i < N / 4; ++i)
    w[i] = __byte_perm(__byte_perm(b[4 * i], b[4 * i + 1], 0x0040u), __byte_perm(b[4 * i + 2], b[4 * i + 3], 0x0040u),
                       0x5410u);
}

// Registers per thread: each SM sub-partition holds a quarter of the register file, and the
// sub-partition with the most warps (the producer's) must fit all of its warps.
constexpr int q8s_max_regs(int ncw) { return (65536 / 4) / (((ncw + 1 + 3) / 4) * 32) / 8 * 8; }

// NB >= 0: the pool keeps n_hp = 16 NB rows in BF16, so a lane's last NB row steps are the
// BF16 rows and every row's kind is known at compile time (no branch per row); NB < 0: any
// even n_hp, each row's kind decided at run time.
template <int RULE, int DK, int DV, typename IT, int NCW, int NB>
__global__ void __launch_bounds__(Q8sCfg<DK, DV, IT, Rule<RULE>::kChannelGate, NCW>::kThreads)
    __maxnreg__(q8s_max_regs(NCW) > 255 ? 255 : q8s_max_regs(NCW)) step_q8s_kernel(const StepParams p) {
  constexpr bool CHG = Rule<RULE>::kChannelGate;
  constexpr bool PRED = Rule<RULE>::kPredicts;
  using C = Q8sCfg<DK, DV, IT, CHG, NCW>;
  constexpr int RL = DK / 16;  // rows per lane
  constexpr int NG = DV / 32;  // 32-column groups per row
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
  griddep_wait();
  griddep_launch_dependents();
#endif

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == NCW) {
    step_producer<RULE, DK, DV, q8_t, IT, false, false, C>(p, smem, meta, full, empty, n_my, lane);
    return;
  }

  const int team = warp / C::kWPT;
  const int part = warp % C::kWPT;
  const int hf = lane & 1;   // half of the warp's 32-column strip (one group)
  const int rb = lane >> 1;  // row block: storage rows 16 m + rb
  const int c0 = part * 32 + hf * 16;
  const int n8 = NB >= 0 ? DK - 16 * NB : DK - p.n_hp;
  float* kp = reinterpret_cast<float*>(smem + C::kOffPerm) + warp * C::kPermFloats;
  float* qp = kp + DK;
  float* ap = qp + DK;
  float* us = ap + DK;  // u of the strip's 32 columns
  unsigned char* dst = static_cast<unsigned char*>(p.dst);
  IT* out = static_cast<IT*>(p.o);

  for (int64_t it = team; it < n_my; it += C::kTeams) {
    const int stage = (int)(it % C::kStages);
    const uint32_t round = (uint32_t)(it / C::kStages);
    const bool arrived = mbar_wait(&full[stage], round & 1u, p.wait_ns);
    if (!__all_sync(0xffffffffu, arrived)) {
      if (lane == 0) report(p.err, LA_DEVERR_TIMEOUT);
      return;
    }
    const StepMeta m = meta[stage];
    if (m.valid) {  // (the same for the whole warp)
      const unsigned char* sb = smem + stage * C::kStageBytes;
      const unsigned char* sc8 = sb + n8 * DV;      // the INT8 block's scales
      const unsigned char* hp = sc8 + n8 * NG * 4;  // the BF16 rows
      const IT* qs = reinterpret_cast<const IT*>(sb + C::kTileBytes);
      const IT* ks = reinterpret_cast<const IT*>(sb + C::kOffK);
      const IT* vs = reinterpret_cast<const IT*>(sb + C::kOffV);
      const float* as = reinterpret_cast<const float*>(sb + C::kOffA);
      float a, bcoef, c;
      Rule<RULE>::coeffs(m.g, m.beta, a, bcoef, c);

      // key, query (and decay) of each storage row, stored lane-major: row 16 m + rb at
      // rb * RL + m.  Lane j places key channels j, j + 32, ...; the producer has checked
      // that the mask marks exactly n_hp rows, so every place is inside the vectors.
      {
        const int h = (int)((blockIdx.x + it * gridDim.x) % H);
        const uint32_t* mk = p.src_mask + h * (DK / 32);
        int below = 0;
#pragma unroll
        for (int w = 0; w < DK / 32; ++w) {
          const uint32_t mw = __ldg(mk + w);
          const int cix = 32 * w + lane;
          const int pre = below + __popc(mw & ((1u << lane) - 1u));
          below += __popc(mw);
          const int vr = ((mw >> lane) & 1u) ? n8 + pre : cix - pre;
          const int pos = (vr & 15) * RL + (vr >> 4);
          kp[pos] = io_load(ks + cix);
          qp[pos] = io_load(qs + cix);
          if (CHG) ap[pos] = as[cix];
        }
        __syncwarp();
      }

      // whether row step ms (storage row 16 ms + rb) is an INT8 row
      auto int8_row = [&](int ms) { return NB >= 0 ? ms < RL - NB : 16 * ms + rb < n8; };
      // a storage row of the lane's 16 columns: values as code, scale (s = 1 for BF16 rows)
      auto load_row = [&](int ms, float* cv, float& s) {
        const int vr = 16 * ms + rb;
        if (int8_row(ms)) {
          const uint4 w = *reinterpret_cast<const uint4*>(sb + vr * DV + c0);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
          q8s_codes<16>(ww, cv);
          s = *reinterpret_cast<const float*>(sc8 + (vr * NG + part) * 4);
        } else {
          const uint4* w = reinterpret_cast<const uint4*>(hp + ((vr - n8) * DV + c0) * 2);
          StateVec<__nv_bfloat16>::unpack(w[0], cv);
          StateVec<__nv_bfloat16>::unpack(w[1], cv + 8);
          s = 1.0f;
        }
      };

      // pass 1: k.q, S^T k and S^T q (kda: the rows' decays scale the keys of both sums)
      float kq = 0.0f, pp[16], rr[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) pp[j] = rr[j] = 0.0f;
#pragma unroll
      for (int m0 = 0; m0 < RL; m0 += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kp + rb * RL + m0);
        const float4 q4 = *reinterpret_cast<const float4*>(qp + rb * RL + m0);
        float4 a4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        if (CHG) a4 = *reinterpret_cast<const float4*>(ap + rb * RL + m0);
        const float kk4[4] = {k4.x, k4.y, k4.z, k4.w}, qq4[4] = {q4.x, q4.y, q4.z, q4.w};
        const float aa4[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int mi = 0; mi < 4; ++mi) {
          float cv[16], s;
          load_row(m0 + mi, cv, s);
          kq = fmaf(kk4[mi], qq4[mi], kq);
          const float k1 = s * (CHG ? kk4[mi] * aa4[mi] : kk4[mi]);
          const float q1 = s * (CHG ? qq4[mi] * aa4[mi] : qq4[mi]);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 c2 = make_float2(cv[j], cv[j + 1]);
            if (PRED) {
              const float2 r2 = __ffma2_rn(c2, make_float2(k1, k1), make_float2(pp[j], pp[j + 1]));
              pp[j] = r2.x;
              pp[j + 1] = r2.y;
            }
            const float2 r3 = __ffma2_rn(c2, make_float2(q1, q1), make_float2(rr[j], rr[j + 1]));
            rr[j] = r3.x;
            rr[j + 1] = r3.y;
          }
        }
      }
      // k.q over the row blocks; the column sums by recursive halving over the row blocks
      // (lane bits 4 .. 1): the values v = (p_0, r_0, p_1, r_1, ...) (without the p when the
      // rule does not predict) halve at each step, and lane (rb, hf) ends with column rb
      // of its half: v[0] = p, v[1] = r (or v[0] = r)
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
      constexpr int NV = PRED ? 32 : 16;
      float v[NV];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (PRED) {
          v[2 * j] = pp[j];
          v[2 * j + 1] = rr[j];
        } else {
          v[j] = rr[j];
        }
      }
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const int half = NV >> (st + 1);
        const bool upper = (rb >> (3 - st)) & 1;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16 >> st);
        }
      }
      const float pcol = PRED ? v[0] : 0.0f;
      const float rcol = PRED ? v[1] : v[0];

      // u = b (v - c p),  o = scale (a r + (k.q) u) of column c0 + rb; u to the warp
      {
        const int col = c0 + rb;
        const float uc = bcoef * (io_load(vs + col) - c * pcol);
        io_store(out + m.o_off + col, p.scale * fmaf(a, rcol, kq * uc));
        us[hf * 16 + rb] = uc;
        __syncwarp();
      }
      float u[16];
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 u4 = *reinterpret_cast<const float4*>(us + hf * 16 + j);
        u[j] = u4.x;
        u[j + 1] = u4.y;
        u[j + 2] = u4.z;
        u[j + 3] = u4.w;
      }

      // pass 2: S' = a S + k u^T, stored in the tile's format at the same storage rows.
      // The fast form takes each group's absmax keeping NaN and converts codes with the
      // float trick; if any INT8 group of the warp held a non-finite value, the whole pass
      // runs again in the codec's form (absmax ignoring NaN, the conversion unit), which
      // overwrites every store of the first run.
      unsigned char* dtile = dst + m.dst_off;
      unsigned char* dsc8 = dtile + n8 * DV;
      unsigned char* dhp = dsc8 + n8 * NG * 4;
      auto pass2 = [&](auto exact_tag) {
        constexpr bool EXACT = decltype(exact_tag)::value;
        bool bad = false;
#pragma unroll
        for (int m0 = 0; m0 < RL; m0 += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kp + rb * RL + m0);
          float4 a4 = make_float4(a, a, a, a);
          if (CHG) a4 = *reinterpret_cast<const float4*>(ap + rb * RL + m0);
          const float kk4[4] = {k4.x, k4.y, k4.z, k4.w}, aa4[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int mi = 0; mi < 4; ++mi) {
            const int ms = m0 + mi;
            const int vr = 16 * ms + rb;
            float cv[16], s;
            load_row(ms, cv, s);
            const float as_ = aa4[mi] * s;
            float y[16];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float2 r2 = __ffma2_rn(make_float2(cv[j], cv[j + 1]), make_float2(as_, as_),
                                           __fmul2_rn(make_float2(kk4[mi], kk4[mi]), make_float2(u[j], u[j + 1])));
              y[j] = r2.x;
              y[j + 1] = r2.y;
            }
            if (int8_row(ms)) {
              // the group's absmax: this lane's 16 values, then the other half's (the two
              // lanes of a row take the same branch; with NB < 0 other rows may not)
              const unsigned pair = NB >= 0 ? 0xffffffffu : 3u << (lane & ~1);
              float amax = 0.0f;
              if (EXACT) {
#pragma unroll
                for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(y[j]));
                amax = fmaxf(amax, __shfl_xor_sync(pair, amax, 1));
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) amax = fmax_nan(amax, fabsf(y[j]));
                amax = fmax_nan(amax, __shfl_xor_sync(pair, amax, 1));
                bad = bad || !(amax <= 3.402823466e38f);
              }
              float sc, inv;
              q8_scales(amax, sc, inv);
              uint32_t w[4];
              if (EXACT) {
                q8_pack<16>(y, inv, w);
              } else {
                q8s_pack<16>(y, inv, w);
              }
              *reinterpret_cast<uint4*>(dtile + vr * DV + c0) = make_uint4(w[0], w[1], w[2], w[3]);
              if (hf == 0) *reinterpret_cast<float*>(dsc8 + (vr * NG + part) * 4) = sc;
            } else {
              uint4* d = reinterpret_cast<uint4*>(dhp + ((vr - n8) * DV + c0) * 2);
              d[0] = StateVec<__nv_bfloat16>::pack(y);
              d[1] = StateVec<__nv_bfloat16>::pack(y + 8);
            }
          }
        }
        return bad;
      };
      if (__any_sync(0xffffffffu, pass2(std::false_type{}))) {
        __syncwarp();  // the first run's stores before the second's (same lanes, same addresses)
        pass2(std::true_type{});
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
  }
}

template <int RULE, int DK, int DV, typename IT, int NB>
cudaError_t launch_step_q8s(const StepParams& p, cudaStream_t stream) {
  constexpr int NCW = LA_Q8S_CONSUMER_WARPS / (DV / 32) * (DV / 32);
  using C = Q8sCfg<DK, DV, IT, Rule<RULE>::kChannelGate, NCW>;
  const void* fn = reinterpret_cast<const void*>(&step_q8s_kernel<RULE, DK, DV, IT, NCW, NB>);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, step_q8s_kernel<RULE, DK, DV, IT, NCW, NB>, p);
  if (e != cudaSuccess) return e;
#else
  step_q8s_kernel<RULE, DK, DV, IT, NCW, NB><<<grid, C::kThreads, C::kSmem, stream>>>(p);
#endif
  return cudaGetLastError();
}

// q8 pools: the storage-order kernel when the source and destination share their mask
// array, the generic step kernel (rows located through each mask) otherwise.
template <int RULE, int DK, int DV, typename IT>
cudaError_t launch_step_q8(const StepParams& p, cudaStream_t stream) {
  if (p.src_mask != p.dst_mask) return launch_step<RULE, DK, DV, q8_t, IT, false>(p, stream);
  // n_hp <= d_k / 4: at most 2 BF16 row steps of 16 rows for d_k = 128, 1 for d_k = 64
  // (with d_k = 64 case 2 cannot occur; were it reached it would fall through to the
  // kernel that decides each row's kind at run time, which takes any even n_hp)
  switch (p.n_hp % 16 == 0 ? p.n_hp / 16 : -1) {
    case 0: return launch_step_q8s<RULE, DK, DV, IT, 0>(p, stream);
    case 1: return launch_step_q8s<RULE, DK, DV, IT, 1>(p, stream);
    case 2: if constexpr (DK >= 128) return launch_step_q8s<RULE, DK, DV, IT, 2>(p, stream);
    default: return launch_step_q8s<RULE, DK, DV, IT, -1>(p, stream);
  }
}

// Launcher table of one io type (each io type in its own translation unit).
template <typename IT>
StepLaunchFn find_step_q8_table(int rule, int dk, int dv) {
#define LA_Q8S_CASE(R, K, V) \
  if (rule == R && dk == K && dv == V) return &launch_step_q8<R, K, V, IT>;
#define LA_Q8S_SHAPES(R) LA_Q8S_CASE(R, 64, 64) LA_Q8S_CASE(R, 128, 64) LA_Q8S_CASE(R, 128, 128)
  LA_Q8S_SHAPES(LA_RULE_LINEAR)
  LA_Q8S_SHAPES(LA_RULE_GATED)
  LA_Q8S_SHAPES(LA_RULE_DELTA)
  LA_Q8S_SHAPES(LA_RULE_GATED_DELTA)
  LA_Q8S_SHAPES(LA_RULE_KDA)
#undef LA_Q8S_SHAPES
#undef LA_Q8S_CASE
  return nullptr;
}

}  // namespace la
