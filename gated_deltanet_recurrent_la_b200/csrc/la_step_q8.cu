// la_step_q8.cu -- decode-step kernels with the mixed INT8 / BF16 (q8) state storage (all
// rules, io dtypes, d_v a multiple of 32): the storage-order kernel of la_step_q8.cuh when
// source and destination share a mask, the generic step kernel of la_step.cuh otherwise.
#include "la_step_q8.cuh"

namespace la {
StepLaunchFn find_step_q8(int rule, int dk, int dv, int io) { return find_step_q8_table(rule, dk, dv, io); }
}  // namespace la
