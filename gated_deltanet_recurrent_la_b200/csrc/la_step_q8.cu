// la_step_q8.cu -- decode-step kernels with the mixed INT8 / BF16 (q8) state storage (all
// rules, io dtypes, d_v a multiple of 32); see la_step.cuh.
#include "la_step.cuh"

namespace la {
StepLaunchFn find_step_q8(int rule, int dk, int dv, int io) { return find_step_q8_impl<false>(rule, dk, dv, io); }
}  // namespace la
