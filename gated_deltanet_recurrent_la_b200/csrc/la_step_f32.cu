// la_step_f32.cu -- decode-step kernels with f32 state storage (all rules, tile shapes
// and io dtypes); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_f32(int rule, int dk, int dv, int io) { return find_step_impl<float, false>(rule, dk, dv, io); }
}  // namespace la
