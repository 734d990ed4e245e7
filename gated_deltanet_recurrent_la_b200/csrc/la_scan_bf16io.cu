// la_scan_bf16io.cu -- scan kernels with bf16 q/k/v/o (all rules and tile shapes); see
// la_scan.cuh.
#include "la_scan.cuh"

namespace la {
ScanLaunchFn find_scan_bf16io(int rule, int dk, int dv) { return find_scan_impl<__nv_bfloat16, false>(rule, dk, dv); }
}  // namespace la
