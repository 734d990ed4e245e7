// la_device.cuh -- device-side building blocks shared by the sm_100a kernels of
// liblastate: shared-memory barriers (mbarrier), 1-D bulk copies global -> shared
// (the TMA engine's cp.async.bulk), 16-byte asynchronous copies, bounded waits and
// BF16 <-> FP32 packing.  Every wait here has a time limit: a wait that gives up
// reports LA_DEVERR_TIMEOUT through the caller's error word instead of hanging.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_state.h"

namespace la {

// Time limit of one pipeline wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s
// Independent cap on the number of polls of one wait.
constexpr uint32_t kWaitMaxPolls = 1u << 26;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report(int32_t* err_word, uint32_t bits) {
  atomicOr(reinterpret_cast<unsigned int*>(err_word), bits);
}

// ---- mbarrier -------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t arrivals) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(arrivals) : "memory");
}

// Makes barrier initialisation visible to the asynchronous (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits until the phase of `bar` with the given parity has completed.  Returns false
// (without reporting) if the time limit (nanoseconds) or the poll cap is reached first.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t polls = 1; polls < kWaitMaxPolls; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((polls & 63u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// ---- bulk copies (TMA engine, no tensor map) ---------------------------------------

// Copies `bytes` (a multiple of 16; both addresses 16-byte aligned) from global to
// this CTA's shared memory; completion is signalled as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Same, with an L2 eviction-priority policy (createpolicy) for data read once.
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---- Ampere-style asynchronous copies (used by the scan's staging) ---------------

__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- programmatic dependent launch ---------------------------------------------------

// Blocks until the preceding kernel on the stream has completed and its memory is
// visible (a no-op when the launch did not allow programmatic overlap).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel on the stream be scheduled (it still waits in griddep_wait).
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// ---- named barriers among a subset of warps ---------------------------------------

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t threads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return out != 0;
}

// ---- BF16 / FP32 ------------------------------------------------------------------
// A bfloat16 is the upper half of an IEEE binary32, so widening is a shift.

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Packs two floats into two bfloat16 (round to nearest even), `a` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T>
struct IoTraits;

template <>
struct IoTraits<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};

template <>
struct IoTraits<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

template <typename T>
__device__ __forceinline__ float io_load(const T* p) { return IoTraits<T>::load(p); }
template <typename T>
__device__ __forceinline__ void io_store(T* p, float x) { IoTraits<T>::store(p, x); }

// 16 bytes of state <-> FP32.  FP32 state: 4 elements per vector; BF16: 8.
template <typename ST>
struct StateVec;

template <>
struct StateVec<float> {
  static constexpr int kElems = 4;
  static __device__ __forceinline__ void unpack(const uint4& w, float* x) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
  }
  static __device__ __forceinline__ uint4 pack(const float* x) {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
  }
};

template <>
struct StateVec<__nv_bfloat16> {
  static constexpr int kElems = 8;
  static __device__ __forceinline__ void unpack(const uint4& w, float* x) {
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
  }
  static __device__ __forceinline__ uint4 pack(const float* x) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
  }
};

// ---- mixed INT8 / BF16 state storage (LA_Q8) ----------------------------------------
// Tile of d_k x d_v: INT8 codes [d_k - n_hp][d_v], FP32 scales [d_k - n_hp][d_v / 32],
// BF16 rows [n_hp][d_v]; the rows whose bit is set in the head's mask (d_k / 32 words)
// are the BF16 ones, each block in increasing row order.  A group of 32 columns of an
// INT8 row with absmax a > 0 has scale s = a * fl(1/127) and inverse scale
// inv = fl(1/a) * 127 (correctly rounded FP32 reciprocal and products); its codes are
// rint(x * inv) clamped to +-127 (NaN -> 0), decoded as code * s; an all-zero group has
// s = inv = 0.
struct q8_t {};

// Rows row0 .. row0 + n - 1 of a head (n <= 32, inside one 32-row word of the mask): each
// row is BF16 (rank among the BF16 rows) or INT8 (rank among the INT8 rows).
template <int DK>
struct Q8Rows {
  uint32_t word;  // the mask word holding the rows
  int below;      // BF16 rows before that word
  int row0;

  __device__ __forceinline__ void init(const uint32_t* head_mask, int first_row) {
    row0 = first_row;
    below = 0;
    word = 0u;
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) {
      const uint32_t m = __ldg(head_mask + w);
      if (w < first_row / 32) below += __popc(m);
      if (w == first_row / 32) word = m;
    }
  }
  // row row0 + r: returns true for a BF16 row; idx = its rank in its block
  __device__ __forceinline__ bool row(int r, int& idx) const {
    const int i = row0 + r, b = i & 31;
    const int pre = below + __popc(word & ((1u << b) - 1u));
    const bool hp = (word >> b) & 1u;
    idx = hp ? pre : i - pre;
    return hp;
  }
};

// scale and inverse scale of a group with absmax `amax` (both 0 for an all-zero group)
__device__ __forceinline__ void q8_scales(float amax, float& s, float& inv) {
  const bool nz = amax > 0.0f;
  s = nz ? __fmul_rn(amax, 1.0f / 127.0f) : 0.0f;
  inv = nz ? __fmul_rn(__frcp_rn(amax), 127.0f) : 0.0f;
}

// The clamp to +-127 never binds here: |x| <= absmax gives |x * inv| <= 127 (1 + 2^-23) <
// 127.5, and the conversion sends NaN to 0, so the conversion alone gives the clamped code.
__device__ __forceinline__ uint32_t q8_code(float x, float inv) {
  return (uint32_t)__float2int_rn(__fmul_rn(x, inv)) & 0xffu;
}

// N (4 or 8) consecutive values <-> codes packed little-endian into N bytes
template <int N>
__device__ __forceinline__ void q8_pack(const float* x, float inv, uint32_t* words) {
#pragma unroll
  for (int w = 0; w < N / 4; ++w)
    words[w] = q8_code(x[4 * w], inv) | (q8_code(x[4 * w + 1], inv) << 8) | (q8_code(x[4 * w + 2], inv) << 16) |
               (q8_code(x[4 * w + 3], inv) << 24);
}

template <int N>
__device__ __forceinline__ void q8_unpack(const uint32_t* words, float s, float* x) {
#pragma unroll
  for (int w = 0; w < N / 4; ++w)
#pragma unroll
    for (int b = 0; b < 4; ++b)
      x[4 * w + b] = __fmul_rn((float)(int)(int8_t)((words[w] >> (8 * b)) & 0xffu), s);
}

// N consecutive io-type values -> FP32, with the widest aligned vector loads the byte
// count allows (16 or 8 bytes; scalar otherwise).  `p` must be aligned to that width.
template <typename IT, int N>
__device__ __forceinline__ void load_f32(const IT* p, float* out) {
  constexpr int kBytes = N * (int)sizeof(IT);
  if constexpr (kBytes % 16 == 0) {
    constexpr int kPer = 16 / sizeof(IT);
#pragma unroll
    for (int i = 0; i < N / kPer; ++i) {
      const uint4 w = reinterpret_cast<const uint4*>(p)[i];
      if constexpr (sizeof(IT) == 2) {
        StateVec<__nv_bfloat16>::unpack(w, out + i * kPer);
      } else {
        StateVec<float>::unpack(w, out + i * kPer);
      }
    }
  } else if constexpr (kBytes % 8 == 0) {
    constexpr int kPer = 8 / sizeof(IT);
#pragma unroll
    for (int i = 0; i < N / kPer; ++i) {
      const uint2 w = reinterpret_cast<const uint2*>(p)[i];
      if constexpr (sizeof(IT) == 2) {
        out[i * kPer + 0] = bf16_lo(w.x); out[i * kPer + 1] = bf16_hi(w.x);
        out[i * kPer + 2] = bf16_lo(w.y); out[i * kPer + 3] = bf16_hi(w.y);
      } else {
        out[i * kPer + 0] = __uint_as_float(w.x); out[i * kPer + 1] = __uint_as_float(w.y);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = io_load(p + i);
  }
}

// N FP32 values -> N consecutive io-type values (BF16 rounded to nearest even).
template <typename IT, int N>
__device__ __forceinline__ void store_f32(IT* p, const float* in) {
  constexpr int kBytes = N * (int)sizeof(IT);
  if constexpr (kBytes % 16 == 0) {
    constexpr int kPer = 16 / sizeof(IT);
#pragma unroll
    for (int i = 0; i < N / kPer; ++i) {
      if constexpr (sizeof(IT) == 2) {
        reinterpret_cast<uint4*>(p)[i] = StateVec<__nv_bfloat16>::pack(in + i * kPer);
      } else {
        reinterpret_cast<uint4*>(p)[i] = StateVec<float>::pack(in + i * kPer);
      }
    }
  } else if constexpr (kBytes % 8 == 0 && sizeof(IT) == 2) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i)
      reinterpret_cast<uint2*>(p)[i] = make_uint2(pack_bf16x2(in[4 * i], in[4 * i + 1]), pack_bf16x2(in[4 * i + 2], in[4 * i + 3]));
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) io_store(p + i, in[i]);
  }
}

// FP32 pair arithmetic.  sm_100 has packed FFMA2 / FMUL2, but in the register-heavy FMA
// loops of these kernels it measured slower on B200 than two scalar FFMAs (identical
// results), so the pairs are computed with scalar instructions unless LA_PACKED_FP32=1.
#ifndef LA_PACKED_FP32
#define LA_PACKED_FP32 0
#endif
__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
#if LA_PACKED_FP32
  return __ffma2_rn(a, b, c);
#else
  return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
#if LA_PACKED_FP32
  return __fmul2_rn(a, b);
#else
  return make_float2(a.x * b.x, a.y * b.y);
#endif
}

// Coefficients (a, b, c) of a rule: S <- a S + k u^T, u = b (v - c S^T k).
// kda (channel-wise gate): the decay is a per-row vector alpha applied to S before the
// prediction, S <- Diag(alpha) S + k u^T with u = beta (v - (Diag(alpha) S)^T k); the
// kernels fold alpha into the keys of the reductions, so its scalar coefficients are
// a = 1 (the readout's S^T q already carries alpha), b = beta, c = 1.
template <int RULE>
struct Rule {
  static constexpr bool kUsesGate = (RULE == LA_RULE_GATED || RULE == LA_RULE_GATED_DELTA);
  static constexpr bool kChannelGate = (RULE == LA_RULE_KDA);
  static constexpr bool kUsesBeta = (RULE == LA_RULE_DELTA || RULE == LA_RULE_GATED_DELTA || RULE == LA_RULE_KDA);
  static constexpr bool kPredicts = kUsesBeta;  // needs S^T k
  static __device__ __forceinline__ void coeffs(float g, float beta, float& a, float& b, float& c) {
    a = kUsesGate ? g : 1.0f;
    b = kUsesBeta ? beta : 1.0f;
    c = (RULE == LA_RULE_DELTA || RULE == LA_RULE_KDA) ? 1.0f : (RULE == LA_RULE_GATED_DELTA ? g : 0.0f);
  }
};

}  // namespace la
