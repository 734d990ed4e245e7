// la_step_conv_bf16.cu -- decode-step kernels with the short causal convolution fused ahead,
// bf16 state storage (all rules, tile shapes and io dtypes); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_conv_bf16(int rule, int dk, int dv, int io) { return find_step_conv_impl<__nv_bfloat16>(rule, dk, dv, io); }
}  // namespace la
