#include "interp_body.cuh"
#include "interp_launch.h"
namespace mk {
const void *spec_kernel_tiny_batched_tqo() {
  return (const void *)interp_kernel<kMaxBatch, false, Spec<32, 32, 8, 2, 2, true>>;
}
}
