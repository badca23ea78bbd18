// The interpreter specialised for hidden 2048, 32 query / 8 KV heads of 64
// (the Llama-3.2-1B shape): 4-row pages for QKV, gate/up, LM head, output and
// down projections.
#include "interp_body.cuh"
#include "interp_launch.h"

namespace mk {
const void *spec_kernel_llama1b() { return (const void *)interp_kernel<1, false, Spec<4, 4, 4, 4, 2>>; }
}  // namespace mk
