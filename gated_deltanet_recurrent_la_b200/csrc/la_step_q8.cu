// la_step_q8.cu -- decode-step kernels with the mixed INT8 / BF16 (q8) state storage (all
// rules, d_v a multiple of 32), BF16 io: the storage-order kernel of la_step_q8.cuh when
// source and destination share a mask, the generic step kernel of la_step.cuh otherwise.
// FP32 io is in la_step_q8_f32io.cu.
#include "la_step_q8.cuh"

namespace la {
StepLaunchFn find_step_q8(int rule, int dk, int dv, int io) {
  return io == LA_F32 ? find_step_q8_f32io(rule, dk, dv) : find_step_q8_table<__nv_bfloat16>(rule, dk, dv);
}
}  // namespace la
