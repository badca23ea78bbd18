// The Llama-3.2-1B-shape interpreter (see interp_spec_llama1b.cu) for batched
// plans: every matrix instruction serves up to kMaxBatch sequences, so each
// weight page is read once per step for all of them.
#include "interp_body.cuh"
#include "interp_launch.h"

namespace mk {
const void *spec_kernel_llama1b_batched() {
  return (const void *)interp_kernel<kMaxBatch, false, Spec<4, 4, 4, 4, 2>>;
}
}  // namespace mk
