// la_scan_f32io.cu -- scan kernels with f32 q/k/v/o (all rules and tile shapes); see
// la_scan.cuh.
#include "la_scan.cuh"

namespace la {
ScanLaunchFn find_scan_f32io(int rule, int dk, int dv) { return find_scan_impl<float, false>(rule, dk, dv); }
}  // namespace la
