// The batched Llama-3.2-1B-shape interpreter (see interp_spec_llama1b_batched.cu)
// with QKV and the O projection as tensor-core tiles too.
#include "interp_body.cuh"
#include "interp_launch.h"

namespace mk {
const void *spec_kernel_llama1b_batched_tqo() {
  return (const void *)interp_kernel<kMaxBatch, false, Spec<4, 4, 4, 4, 2, true>>;
}
}  // namespace mk
