// Host-side entry points of the interpreter kernels.  The shape-generic
// kernel (and the raw-layout variant) live in interp.cu; each shape-
// specialised kernel is built in its own translation unit so that the
// builds compile in parallel.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

#include "mk_internal.h"

namespace mk {
// Dynamic shared memory of a CTA with `num_pages` ring pages and a staging
// region of `act_floats` floats.
int shared_bytes_fixed(int num_pages, size_t act_floats);
// Floats of the staging region for a model shape and `nb` sequences per
// instruction (1, or kMaxBatch for batched builds): input vectors or the
// split-page partial table and the O projection's residual rows, the
// attention scratch, and in batched builds the tensor-core exchange.
size_t staging_floats(int H, int qdim, int KCd, int G, int d, int nb);
// Ring pages that fit next to a staging region of `act_floats` floats in
// `smem_optin` bytes: a multiple of the loader count with twice it a
// multiple of the compute-warp count (unambiguous mbarrier phases), at most
// 16; 0 if fewer than 2 * kLoaders fit.
int ring_pages(int smem_optin, size_t act_floats);
// The interpreter kernel for the model shape in p and `nb` sequences per
// instruction (1, or kMaxBatch for batched plans): a shape-specialised build
// when one exists and `specialised` is set (*variant = 1), else the
// shape-generic one (*variant = 0).  Batched plans have specialised builds
// only (`tqo`: the build with QKV and the O projection on the tensor cores);
// nullptr when the shape has none.
const void *interp_kernel_for(const KParams &p, bool specialised, int nb, bool tqo, int *variant);
// The raw-layout variant (weights read in the caller's layout).
const void *interp_kernel_raw();
// the tensor-parallel rank build (shape-generic, batch 1, static queues)
const void *interp_kernel_tp();
// Allow `smem` bytes of dynamic shared memory for fn and report how many of
// its CTAs fit on one SM.
cudaError_t interp_prepare(const void *fn, int smem, int *blocks_per_sm);
// Launch fn over `grid` CTAs (cooperatively when asked).
cudaError_t launch_interp(const void *fn, const KParams &p, int grid, int smem, cudaStream_t st, bool cooperative);

// shape-specialised kernels (interp_spec_*.cu)
const void *spec_kernel_llama1b();
const void *spec_kernel_llama1b_batched();
const void *spec_kernel_llama1b_batched_tqo();
const void *spec_kernel_llama8b();
}  // namespace mk
