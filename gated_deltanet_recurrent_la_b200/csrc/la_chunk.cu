// la_chunk.cu -- chunked tensor-core prefill kernels: the fused one-launch form (the four
// scalar-gate rules, la_chunk_fused.cuh), the two-launch form of the delta rules
// (la_chunk.cuh prep + la_chunk_tc.cuh recurrence) and the two-launch form of the
// channel-wise gate (la_chunk_kda.cuh).
#include "la_chunk.cuh"
#include "la_chunk_conv.cuh"
#include "la_chunk_fused.cuh"
#include "la_chunk_kda.cuh"
#include "la_chunk_tc.cuh"

namespace la {
ScanLaunchFn find_chunk_scan(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_fused<LA_RULE_LINEAR>;
    case LA_RULE_GATED: return &launch_chunk_fused<LA_RULE_GATED>;
    case LA_RULE_DELTA: return &launch_chunk_fused<LA_RULE_DELTA>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_fused<LA_RULE_GATED_DELTA>;
  }
  return nullptr;
}
// The query-group direction: the one-launch form once per query of the group, each launch
// writing its query head's outputs; the state (the same in every launch) is written by the
// launch of query 0, which runs last (a read slot may be the write slot).
template <int RULE>
cudaError_t launch_chunk_qgroups(const ScanParams& p, cudaStream_t stream) {
  for (int qi = p.q_group - 1; qi >= 0; --qi) {
    ScanParams f = p;
    f.q_index = qi;
    const cudaError_t e = launch_chunk_fused<RULE, false>(f, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}
ScanLaunchFn find_chunk_scan_qgroups(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_qgroups<LA_RULE_LINEAR>;
    case LA_RULE_GATED: return &launch_chunk_qgroups<LA_RULE_GATED>;
    case LA_RULE_DELTA: return &launch_chunk_qgroups<LA_RULE_DELTA>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_qgroups<LA_RULE_GATED_DELTA>;
  }
  return nullptr;
}
ScanLaunchFn find_chunk_scan_conv(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_fused<LA_RULE_LINEAR, true>;
    case LA_RULE_GATED: return &launch_chunk_fused<LA_RULE_GATED, true>;
    case LA_RULE_DELTA: return &launch_chunk_fused<LA_RULE_DELTA, true>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_fused<LA_RULE_GATED_DELTA, true>;
  }
  return nullptr;
}
// The convolution as a launch of its own (every tile in parallel, its output through the
// workspace), then the one-launch chunked kernel on the convolved q, k, v (one q/k head per
// state head: the convolution's histories are per state head).
template <int RULE>
cudaError_t launch_chunk_conv_ws(const ScanParams& p, cudaStream_t stream) {
  if (p.n_seqs <= 0) return cudaSuccess;
  const void* fn = reinterpret_cast<const void*>(&chunk_conv_kernel);
  const int per_sm = prepare_kernel(fn, cconv::kThreads, cconv::kSmem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  chunk_conv_kernel<<<device_sm_count() * per_sm, cconv::kThreads, cconv::kSmem, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ScanParams f = p;
  const __nv_bfloat16* planes =
      static_cast<const __nv_bfloat16*>(p.workspace) + cconv::kWsHeadBytes / 2;
  const int64_t plane = (int64_t)p.total_tokens * p.n_v_heads * cconv::kD;
  f.q = planes;
  f.k = planes + plane;
  f.v = planes + 2 * plane;
  f.n_qk_heads = p.n_v_heads;
  f.conv_w = 0;
  return launch_chunk_fused<RULE, false>(f, stream);
}
ScanLaunchFn find_chunk_scan_conv_ws(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_conv_ws<LA_RULE_LINEAR>;
    case LA_RULE_GATED: return &launch_chunk_conv_ws<LA_RULE_GATED>;
    case LA_RULE_DELTA: return &launch_chunk_conv_ws<LA_RULE_DELTA>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_conv_ws<LA_RULE_GATED_DELTA>;
  }
  return nullptr;
}
size_t chunk_conv_workspace_bytes(int64_t total_tokens, int64_t n_v_heads) {
  return chunk_conv_workspace_bytes_impl(total_tokens, n_v_heads);
}
size_t chunk_workspace_bytes(int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads) {
  if (total_tokens < 0 || n_seqs < 0 || n_v_heads <= 0) return 0;
  const int64_t tiles = (total_tokens + chunk::kC - 1) / chunk::kC + n_seqs + 1;
  return (size_t)(chunk::kWsHeadBytes + tiles * n_v_heads * chunk::kPrepTileBytes);
}

// The delta rules: the intra-chunk inverses of every chunk (parallel launch), then the
// recurrence on the fifth-generation tensor cores reading them.
template <int RULE>
cudaError_t launch_chunk_scan_ws_tc(const ScanParams& p, cudaStream_t stream) {
  cudaError_t e = launch_chunk_prep<RULE>(p, stream);
  if (e != cudaSuccess) return e;
  return launch_chunk_tc<RULE>(p, stream);
}

ScanLaunchFn find_chunk_scan_ws(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_fused<LA_RULE_LINEAR>;  // no inverse, no workspace
    case LA_RULE_GATED: return &launch_chunk_fused<LA_RULE_GATED>;
    case LA_RULE_DELTA: return &launch_chunk_scan_ws_tc<LA_RULE_DELTA>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_scan_ws_tc<LA_RULE_GATED_DELTA>;
    case LA_RULE_KDA: return &launch_chunk_kda;
  }
  return nullptr;
}
size_t chunk_kda_workspace_bytes(int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads) {
  return kda_workspace_bytes(total_tokens, n_seqs, n_v_heads);
}
}  // namespace la
