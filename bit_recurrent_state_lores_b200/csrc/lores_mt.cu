// lores_mt.cu -- multi-token decode-step kernels (T consecutive tokens per launch), in a
// translation unit of their own so that the two kernel families compile in parallel.
#include "lores_step.cuh"

namespace lores {

StepFn mt_step_kernel_for(int dk, bool diag, bool delta, bool sr) {
  return pick_step_any<true>(dk, diag, delta, sr);
}

}  // namespace lores
