// lores_inst.cu -- one family of decode-step kernels for one key width, compiled once per
// (LORES_DK, LORES_MT, LORES_EXT) so that the families build in parallel:
//   LORES_MT  = 1: multi-token steps (lores_decode_steps); 0: single-token steps
//   LORES_EXT = 1: with the dense 5- to 7-bit and per-lane (per-channel) storage paths
// The function defined here returns the kernel for the decay/delta/rounding modes.
#include "lores_step.cuh"

#if !defined(LORES_DK) || !defined(LORES_MT) || !defined(LORES_EXT)
#error "compile with -DLORES_DK=<16|32|64|128|256> -DLORES_MT=<0|1> -DLORES_EXT=<0|1>"
#endif

#define LORES_CAT2(a, b, c, d) a##_##b##_##c##_##d
#define LORES_CAT(a, b, c, d) LORES_CAT2(a, b, c, d)

namespace lores {

StepFn LORES_CAT(step_kernels, LORES_DK, LORES_MT, LORES_EXT)(bool diag, bool delta, bool sr) {
  return sr ? pick_step<LORES_DK, true, LORES_MT != 0, LORES_EXT != 0>(diag, delta)
            : pick_step<LORES_DK, false, LORES_MT != 0, LORES_EXT != 0>(diag, delta);
}

}  // namespace lores
