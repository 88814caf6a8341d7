// lores_inst.cu -- one family of decode-step kernels for one key width, compiled once per
// family so that the families build in parallel:
//   -DLORES_DK=<d_k> -DLORES_MT=<0|1> -DLORES_EXT=<0|1>: the value-axis step kernels
//     LORES_MT  = 1: multi-token steps (lores_decode_steps); 0: single-token steps
//     LORES_EXT = 1: with the dense 5- to 7-bit and per-lane (per-channel) storage paths
//     LORES_EXT = 2: with the per-lane path only
//     LORES_EXT = 3: the plain kernel with the exact contractions (byte and nibble heads
//                    with one scale per row)
//     LORES_EXT = 4: the dense and per-lane paths with the exact contractions
//   -DLORES_DK=<d_k> -DLORES_KEY=1: the key-axis step and loader kernels
//   -DLORES_DK=<d_k> -DLORES_PAIR=1 -DLORES_MT=<0|1>: the two-rows-per-lane step kernels
//     (heads of one byte or one nibble per code, several scales per row), single- or
//     multi-token
//   -DLORES_DK=<d_k> -DLORES_MMA=1: the tensor-core step kernels (heads of one byte or one
//     nibble per code, one scale per row), single- and multi-token
// The function defined here returns the kernel for the requested modes.
#include "lores_step.cuh"
#include "lores_key.cuh"
#include "lores_pair.cuh"
#include "lores_mma.cuh"

#define LORES_CAT2(a, b, c, d) a##_##b##_##c##_##d
#define LORES_CAT(a, b, c, d) LORES_CAT2(a, b, c, d)
#define LORES_CAT1_2(a, b) a##_##b
#define LORES_CAT1(a, b) LORES_CAT1_2(a, b)
#define LORES_CAT3_2(a, b, c) a##_##b##_##c
#define LORES_CAT3(a, b, c) LORES_CAT3_2(a, b, c)

namespace lores {

#if defined(LORES_PAIR)
#if !defined(LORES_DK)
#error "compile with -DLORES_DK=<16|32|64|128|256> -DLORES_PAIR=1"
#endif
#if !defined(LORES_MT)
#error "compile with -DLORES_DK=<16|32|64|128|256> -DLORES_PAIR=1 -DLORES_MT=<0|1>"
#endif
StepFn LORES_CAT3(pair_kernels, LORES_DK, LORES_MT)(bool diag, bool delta, bool sr) {
  constexpr bool kMT = LORES_MT != 0;
  return sr ? pick_pair<LORES_DK, true, false, kMT>(diag, delta)
            : pick_pair<LORES_DK, false, false, kMT>(diag, delta);
}
#elif defined(LORES_MMA)
#if !defined(LORES_DK)
#error "compile with -DLORES_DK=<16|32|64|128> -DLORES_MMA=1"
#endif
StepFn LORES_CAT1(mma_kernels, LORES_DK)(bool diag, bool delta, bool sr, bool mt) {
  if (mt) return sr ? pick_mma<LORES_DK, true, true>(diag, delta) : pick_mma<LORES_DK, false, true>(diag, delta);
  return sr ? pick_mma<LORES_DK, true, false>(diag, delta) : pick_mma<LORES_DK, false, false>(diag, delta);
}
#elif defined(LORES_KEY)
#if !defined(LORES_DK)
#error "compile with -DLORES_DK=<16|32|64|128|256> -DLORES_KEY=1"
#endif
KeyFn LORES_CAT1(key_kernels, LORES_DK)(bool sr, bool load) {
  if (load)
    return sr ? decode_step_key_kernel<LORES_DK, true, true>
              : decode_step_key_kernel<LORES_DK, false, true>;
  return sr ? decode_step_key_kernel<LORES_DK, true, false>
            : decode_step_key_kernel<LORES_DK, false, false>;
}
#else
#if !defined(LORES_DK) || !defined(LORES_MT) || !defined(LORES_EXT)
#error "compile with -DLORES_DK=<16|32|64|128|256> -DLORES_MT=<0|1> -DLORES_EXT=<0|1|2|3|4>"
#endif
StepFn LORES_CAT(step_kernels, LORES_DK, LORES_MT, LORES_EXT)(bool diag, bool delta, bool sr) {
  return sr ? pick_step<LORES_DK, true, LORES_MT != 0, LORES_EXT>(diag, delta)
            : pick_step<LORES_DK, false, LORES_MT != 0, LORES_EXT>(diag, delta);
}
#endif

}  // namespace lores
