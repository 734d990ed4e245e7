// la_chunk.cu -- chunked tensor-core prefill kernels: the fused one-launch form (the four
// scalar-gate rules, la_chunk_fused.cuh), the two-launch form of the delta rules
// (la_chunk.cuh prep + la_chunk_tc.cuh recurrence) and the two-launch form of the
// channel-wise gate (la_chunk_kda.cuh).
#include "la_chunk.cuh"
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
ScanLaunchFn find_chunk_scan_conv(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_fused<LA_RULE_LINEAR, true>;
    case LA_RULE_GATED: return &launch_chunk_fused<LA_RULE_GATED, true>;
    case LA_RULE_DELTA: return &launch_chunk_fused<LA_RULE_DELTA, true>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_fused<LA_RULE_GATED_DELTA, true>;
  }
  return nullptr;
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
