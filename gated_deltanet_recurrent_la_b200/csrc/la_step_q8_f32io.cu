// la_step_q8_f32io.cu -- the q8 decode-step kernels of la_step_q8.cuh with FP32 io.
#include "la_step_q8.cuh"

namespace la {
StepLaunchFn find_step_q8_f32io(int rule, int dk, int dv) { return find_step_q8_table<float>(rule, dk, dv); }
}  // namespace la
