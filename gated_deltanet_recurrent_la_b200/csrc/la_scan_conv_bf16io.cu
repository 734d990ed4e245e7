// la_scan_conv_bf16io.cu -- scan kernels with the short causal convolution ahead of every token,
// bf16 q/k/v/o (all rules and tile shapes); see la_scan.cuh.
#include "la_scan.cuh"

namespace la {
ScanLaunchFn find_scan_conv_bf16io(int rule, int dk, int dv) { return find_scan_conv_impl<__nv_bfloat16>(rule, dk, dv); }
}  // namespace la
