// la_chunk.cu -- chunked tensor-core prefill kernels (all four rules); see la_chunk.cuh.
#include "la_chunk.cuh"

namespace la {
ScanLaunchFn find_chunk_scan(int rule) {
  switch (rule) {
    case LA_RULE_LINEAR: return &launch_chunk_scan<LA_RULE_LINEAR>;
    case LA_RULE_GATED: return &launch_chunk_scan<LA_RULE_GATED>;
    case LA_RULE_DELTA: return &launch_chunk_scan<LA_RULE_DELTA>;
    case LA_RULE_GATED_DELTA: return &launch_chunk_scan<LA_RULE_GATED_DELTA>;
  }
  return nullptr;
}
}  // namespace la
