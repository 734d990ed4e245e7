// la_step_qg_f32.cu -- decode-step kernels in the query-group direction with f32 state storage (all
// rules, tile shapes and io dtypes); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_qgroups_f32(int rule, int dk, int dv, int io) {
  return find_step_impl<float, true>(rule, dk, dv, io);
}
}  // namespace la
