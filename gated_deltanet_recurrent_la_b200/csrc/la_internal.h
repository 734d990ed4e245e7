// la_internal.h -- host-side interfaces between the C-ABI layer (la_api.cu) and the
// kernel families (step, scan, pool).  Not installed; not part of the ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "la_state.h"

namespace la {

// Bytes of one (slot, head) tile of the mixed INT8 / BF16 (q8) storage: INT8 codes and
// FP32 scales (one per 32 columns) of the d_k - n_hp INT8 rows, then n_hp BF16 rows.
__host__ __device__ constexpr int64_t q8_tile_bytes(int dk, int dv, int n_hp) {
  return (int64_t)(dk - n_hp) * dv + (int64_t)(dk - n_hp) * (dv / 32) * 4 + (int64_t)n_hp * dv * 2;
}

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
  int32_t q_group;          // queries per state head: 1, or up to 8 in the query-group direction
  int32_t n_hp;             // q8 pools: BF16 key channels per head (same for source and destination)
  const uint32_t* src_mask; // q8 pools: [H_v][d_k / 32] channel masks
  const uint32_t* dst_mask;
  // the short causal convolution ahead of the step (conv_w == 0: none)
  int32_t conv_w;
  int32_t conv_act;         // 1: SiLU
  int32_t conv_l2norm;      // 1: q and k to unit length
  const float* conv_wq;     // [H_qk][d_k][W]
  const float* conv_wk;
  const float* conv_wv;     // [H_v][d_v][W]
  const void* conv_src;     // io dtype [src slots][H_v][2 d_k + d_v][W - 1]
  void* conv_dst;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float scale;
  void* o;
  int32_t* err;
  // failure-path test hooks: the time limit of every pipeline wait (ns), and a tile whose
  // arrival the producer of CTA 0 withholds (-1: none) so that its consumers' waits expire
  uint64_t wait_ns;
  int64_t withhold;
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
  int32_t q_group;           // queries per state head: 1, or up to 8 in the query-group direction
  int32_t q_index;           // chunked prefill in the query-group direction: the query of the group
                             // this launch reads (the state is written by query 0 alone)
  int32_t src_n_hp;          // q8 pools: BF16 key channels per head and the channel masks
  const uint32_t* src_mask;
  int32_t dst_n_hp;
  const uint32_t* dst_mask;
  // the short causal convolution ahead of every token (conv_w == 0: none)
  int32_t conv_w;
  int32_t conv_act;
  int32_t conv_l2norm;
  const float* conv_wq;
  const float* conv_wk;
  const float* conv_wv;
  const void* conv_src;     // io dtype [src slots][H_v][2 d_k + d_v][W - 1]
  void* conv_dst;
  const void* workspace;     // chunked prefill in two launches: the per-chunk Tw / Tu tiles
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

// Decode step with the short causal convolution fused ahead (widths 2 .. kMaxConvWidth).
constexpr int kMaxConvWidth = 4;
StepLaunchFn find_step_conv_f32(int rule, int dk, int dv, int io);
StepLaunchFn find_step_conv_bf16(int rule, int dk, int dv, int io);
ScanLaunchFn find_scan_conv_f32io(int rule, int dk, int dv);
ScanLaunchFn find_scan_conv_bf16io(int rule, int dk, int dv);

// The same in the query-group direction (k per state head, q_group <= kMaxQueryGroup
// query heads reading each state head).
constexpr int kMaxQueryGroup = 8;
// q8 state storage (d_v a multiple of 32): (64,64), (128,64), (128,128)
StepLaunchFn find_step_q8(int rule, int dk, int dv, int io);
StepLaunchFn find_step_q8_f32io(int rule, int dk, int dv);
StepLaunchFn find_step_qgroups_f32(int rule, int dk, int dv, int io);
StepLaunchFn find_step_qgroups_bf16(int rule, int dk, int dv, int io);
ScanLaunchFn find_scan_qgroups_f32io(int rule, int dk, int dv);
ScanLaunchFn find_scan_qgroups_bf16io(int rule, int dk, int dv);

// Chunked tensor-core prefill (d_k = d_v = 128, BF16 io); nullptr for a rule without it.
// The _ws form runs the intra-chunk part as a separate launch through ScanParams::workspace
// (the delta rules and kda; kda has only this form).
ScanLaunchFn find_chunk_scan(int rule);
ScanLaunchFn find_chunk_scan_ws(int rule);
// the one-launch form in the query-group direction (scalar-gate rules)
ScanLaunchFn find_chunk_scan_qgroups(int rule);
// the one-launch form with the short causal convolution ahead (scalar-gate rules), and the
// two-launch form (the convolution's output through a workspace of
// chunk_conv_workspace_bytes(T, H_v) bytes)
ScanLaunchFn find_chunk_scan_conv(int rule);
ScanLaunchFn find_chunk_scan_conv_ws(int rule);
size_t chunk_conv_workspace_bytes(int64_t total_tokens, int64_t n_v_heads);
// workspace of the _ws form: one tile per (chunk slot, head), 17.9 KB for the delta rules,
// 65 KB for kda
size_t chunk_workspace_bytes(int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads);
size_t chunk_kda_workspace_bytes(int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads);
// the library's own fixed workspace on the current device: *addr = its device address,
// *bytes = its size; the error of the device query or the symbol lookup otherwise
cudaError_t chunk_noalloc_workspace(void** addr, size_t* bytes);

cudaError_t launch_pool_copy(const PoolCopyParams& p, cudaStream_t stream);

// FP32 dense tiles <-> q8 slots of a pool (n slots x H_v heads).
struct Q8CodecParams {
  void* pool;                // q8 pool data
  int32_t n_slots;
  int32_t n_v_heads, d_k, d_v, n_hp;
  const uint32_t* mask;      // [H_v][d_k / 32]
  const int32_t* slots;      // [n]
  int32_t n;
  float* dense;              // [n, H_v, d_k, d_v]
  int32_t encode;            // 1: dense -> pool, 0: pool -> dense
  int32_t* err;
};
cudaError_t launch_q8_codec(const Q8CodecParams& p, cudaStream_t stream);

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Resident CTAs per SM of `func` for the given block size / dynamic shared memory,
// after raising the function's dynamic shared-memory limit on the current device.
// Cached per (func, device).  Returns 0 on failure.
int prepare_kernel(const void* func, int threads, int smem_bytes);

}  // namespace la
