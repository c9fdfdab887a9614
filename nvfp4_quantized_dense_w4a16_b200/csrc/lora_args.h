// Arguments of a LoRA delta applied in a projection's epilogue.
#pragma once

#include <stdint.h>

namespace ffn {

// delta[j, n] = sum_i xa[j, off + i] * B[n, i] over the rank r (i ascending,
// fp32), added to the projection's bf16 output and rounded to bf16 again.
// b0 is the gate (or the only) adapter's B, b1 the up adapter's for a fused
// gate+up projection; null pointers mean no adapter.
struct LoraArgs {
  const uint16_t* xa = nullptr;  // [m, xa_ld] bf16: the rank-r products x A^T
  int xa_ld = 0;
  const uint16_t* b0 = nullptr;  // [rows, r] bf16
  const uint16_t* b1 = nullptr;
  int off0 = 0, off1 = 0;        // columns of xa holding each adapter's product
  int r = 0;
};

}  // namespace ffn
