// la_internal.h -- host-side interfaces between the C-ABI layer (la_api.cu) and the
// kernel families (step, scan, pool).  Not installed; not part of the ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "la_state.h"

namespace la {

struct StepParams {
  const void* src;          // source pool data
  int32_t src_slots;
  void* dst;                // destination pool data
  int32_t dst_slots;
  const int32_t* read_slot;   // [B] or nullptr
  const int32_t* write_slot;  // [B] or nullptr
  int32_t B;
  int32_t n_qk_heads;
  int32_t n_v_heads;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float scale;
  void* o;
  int32_t* err;
};

struct ScanParams {
  const void* src;           // source pool or nullptr
  int32_t src_slots;
  int32_t src_dtype;         // la_dtype of src
  const int32_t* read_slot;  // [n_seqs] or nullptr (zero initial state)
  void* dst;
  int32_t dst_slots;
  int32_t dst_dtype;
  const int32_t* write_slot;  // [n_seqs] or nullptr
  int32_t n_seqs;
  const int32_t* cu_seqlens;
  int32_t total_tokens;
  const int32_t* seq_order;  // [n_seqs] or nullptr
  int32_t n_qk_heads;
  int32_t n_v_heads;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float scale;
  void* o;
  int32_t* err;
  int32_t ckpt_every;          // > 0: intermediate states every ckpt_every tokens
  const int32_t* ckpt_cu;      // [n_seqs + 1] offsets into ckpt_slots
  const int32_t* ckpt_slots;   // destination slots of the checkpoints
};

struct PoolCopyParams {
  const void* src;            // source base
  const int32_t* src_index;   // [n] or nullptr (identity)
  int32_t src_count;          // number of valid source slots
  void* dst;                  // destination base
  const int32_t* dst_index;   // [n] or nullptr (identity)
  int32_t dst_count;
  int32_t n;                  // slots to move
  int64_t slot_bytes;         // multiple of 16
  int32_t zero;               // 1: write zeros instead of copying
  int32_t* err;
};

using StepLaunchFn = cudaError_t (*)(const StepParams&, cudaStream_t);
using ScanLaunchFn = cudaError_t (*)(const ScanParams&, cudaStream_t);

// Launchers for a (rule, d_k, d_v, io dtype) of the given state dtype; nullptr when the
// combination is not compiled.
StepLaunchFn find_step_f32(int rule, int dk, int dv, int io);
StepLaunchFn find_step_bf16(int rule, int dk, int dv, int io);
ScanLaunchFn find_scan_f32io(int rule, int dk, int dv);
ScanLaunchFn find_scan_bf16io(int rule, int dk, int dv);

// Chunked tensor-core prefill (d_k = d_v = 128, BF16 io); nullptr for an unknown rule.
ScanLaunchFn find_chunk_scan(int rule);

cudaError_t launch_pool_copy(const PoolCopyParams& p, cudaStream_t stream);

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Resident CTAs per SM of `func` for the given block size / dynamic shared memory,
// after raising the function's dynamic shared-memory limit on the current device.
// Cached per (func, device).  Returns 0 on failure.
int prepare_kernel(const void* func, int threads, int smem_bytes);

}  // namespace la
