// la_step_qg_bf16.cu -- decode-step kernels in the query-group direction with bf16 state storage (all
// rules, tile shapes and io dtypes); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_qgroups_bf16(int rule, int dk, int dv, int io) {
  return find_step_impl<__nv_bfloat16, true>(rule, dk, dv, io);
}
}  // namespace la
