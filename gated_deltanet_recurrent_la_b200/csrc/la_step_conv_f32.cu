// la_step_conv_f32.cu -- decode-step kernels with the short causal convolution fused ahead,
// f32 state storage (all rules, tile shapes and io dtypes); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_conv_f32(int rule, int dk, int dv, int io) { return find_step_conv_impl<float>(rule, dk, dv, io); }
}  // namespace la
