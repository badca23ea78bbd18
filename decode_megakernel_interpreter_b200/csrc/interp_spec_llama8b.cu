// The interpreter specialised for hidden 4096, 32 query / 8 KV heads of 128
// (the Llama-3.1-8B shape): 2-row pages for QKV, gate/up, LM head and output
// projection, 4-row pages for the down projection; batch-1 matrix pages are
// split across the compute warps (split pages).
#include "interp_body.cuh"
#include "interp_launch.h"

namespace mk {
const void *spec_kernel_llama8b() { return (const void *)interp_kernel<1, false, Spec<2, 2, 4, 4, 4, false, true>>; }
}  // namespace mk
