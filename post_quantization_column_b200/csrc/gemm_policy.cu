// gemm_policy.cu — which form of the loss GEMM a search runs (host side): the one-SM or
// the two-SM kernel, the reference output in the candidates' launch or in its own, and
// the candidate operands from qdq_kernel or from the GEMM's own QDQ warps. Each choice
// states the measurement it rests on and the environment variable that overrides it.
#include "awq_kernels.h"

#include <cstdlib>
#include <cstring>

namespace awq {

// The one-SM kernel runs by default for every size: measured on one B200 (median of
// repeated searches, candidate-GEMM phase) it is as fast as the pair kernel on the 4096^3
// layer (1.954 vs 1.967 ms) and faster on the 7B down projection (5.22 vs 5.46 ms), the
// 7B gate+up layer (10.7 vs 10.9 ms) and the 70B gate+up layer (259 vs 342 ms, where
// the pair kernel's clock falls further under the 1 kW power cap). AWQ_GEMM_VARIANT=2
// selects the pair kernel.
int gemm_variant(int64_t M, int64_t K, int64_t N, int n_grid) {
  (void)M;
  (void)K;
  (void)N;
  (void)n_grid;
  const char* v = getenv("AWQ_GEMM_VARIANT");
  return (v && v[0] == '2') ? 2 : 1;
}

// Measured on one B200 (the candidate-GEMM phases, reference launch included, median of 15
// searches per form, interleaved): on the 70B gate+up layer (Y 3.76 GB) the two launches
// with the candidate-inner walk took 249.6 ms against 257.8 ms for the one mode-4 launch
// (its candidates read Y from DRAM once each, 75 GB per search); on the 7B gate+up layer
// (Y 361 MB) 11.37 against 11.56 ms; on the 4096^3 layer (Y 67 MB, held in L2 by the
// mode-4 walk) 2.047 against 2.033 ms, so mode 4 stays below the L2 size. The candidate-
// inner walk inside the one mode-4 launch lost instead: its candidate tiles then wait for
// reference tiles computed in the same wave, and the static tile-to-CTA assignment lets
// CTAs drift apart by many tiles over a launch.
// AWQ_REFERENCE_LAUNCH=own or =fused in the environment selects a form at every size.
bool reference_in_own_launch(int64_t M, int64_t N, int l2_bytes) {
  const char* f = getenv("AWQ_REFERENCE_LAUNCH");
  if (f && !strcmp(f, "own")) return true;
  if (f && !strcmp(f, "fused")) return false;
  return M * N * 4 > static_cast<int64_t>(l2_bytes);
}

// Measured on one B200 (whole searches, median of 12 per form, interleaved on one box):
// with the QDQ warps against qdq_kernel first, 2.41 against 2.46 ms on the 4096^3 layer,
// 13.04 against 13.76 ms on the 7B gate+up layer and 6.35 against 6.78 ms on the 7B down
// projection; on the 70B gate+up layer (308 TFLOP of candidate GEMM work) 272.7 against
// 271.4 ms. That search runs at the 1 kW power cap for its whole length, so the QDQ's
// energy costs the GEMM the same time whether the two overlap or not; from 100 TFLOP of
// candidate GEMM work on, qdq_kernel runs first and the loss GEMM's launches hold only
// the GEMM.
bool qdq_in_loss_gemm(int in_dtype, int group, int variant, int64_t M, int64_t K, int64_t N, int n_grid) {
  const char* f = getenv("AWQ_QDQ");
  if (f && !strcmp(f, "standalone")) return false;
  const bool possible = in_dtype == 0 /* bf16 */ && group == 128 && variant == 1;
  if (f && !strcmp(f, "warps")) return possible;
  return possible && 2.0 * static_cast<double>(M) * K * N * n_grid < 1e14;
}

}  // namespace awq
