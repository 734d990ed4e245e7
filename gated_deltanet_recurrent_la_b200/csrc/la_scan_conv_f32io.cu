// la_scan_conv_f32io.cu -- scan kernels with the short causal convolution ahead of every token,
// f32 q/k/v/o (all rules and tile shapes); see la_scan.cuh.
#include "la_scan.cuh"

namespace la {
ScanLaunchFn find_scan_conv_f32io(int rule, int dk, int dv) { return find_scan_conv_impl<float>(rule, dk, dv); }
}  // namespace la
