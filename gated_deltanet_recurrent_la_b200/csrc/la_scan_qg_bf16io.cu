// la_scan_qg_bf16io.cu -- scan kernels in the query-group direction with bf16 q/k/v/o (all rules and tile
// shapes); see la_scan.cuh.
#include "la_scan.cuh"

namespace la {
ScanLaunchFn find_scan_qgroups_bf16io(int rule, int dk, int dv) { return find_scan_impl<__nv_bfloat16, true>(rule, dk, dv); }
}  // namespace la
