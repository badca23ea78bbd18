// The decode interpreter's host entry: kernel selection and launch.  The
// device code is in interp_body.cuh.
#include <algorithm>

#include "interp_body.cuh"
#include "interp_launch.h"

namespace mk {

int shared_bytes_fixed(int num_pages, size_t act_floats) {
  return (int)((size_t)num_pages * kPageBytes + act_floats * 4 + (size_t)num_pages * 16 + sizeof(Shared) +
               34 * sizeof(int) + 64);
}

size_t staging_floats(int H, int qdim, int KCd, int G, int d, int nb) {
  // input vector per sequence (batch 1: also the O projection's residual rows
  // after the vector, or after the split-page partial table)
  size_t vec = nb == 1 ? std::max({(size_t)H, (size_t)qdim + H, (size_t)KCd, (size_t)kSplitRedFloats + H})
                       : (size_t)nb * std::max({H, qdim, KCd});
  // warps' partials + the current K/V rows (bf16) + the warps' merge weights
  // (+ batched builds: two K and two V rows of a prompt chunk per warp, bf16)
  size_t attn = (size_t)kComputeWarps * G * (d + 2) + (size_t)d + (((size_t)G * (kComputeWarps + 2) + 3) & ~(size_t)3) +
                (nb > 1 ? (size_t)kComputeWarps * 2 * d : 0);
  size_t f = std::max(vec, attn);
  // batched builds: the tensor-core epilogue exchange follows the staged vectors
  if (nb > 1) f += kTcXchFloats;
  return (f + 31) / 32 * 32;
}

int ring_pages(int smem_optin, size_t act_floats) {
  int n = (smem_optin - shared_bytes_fixed(0, act_floats)) / (kPageBytes + 16);
  n = std::min(n, 16) / kLoaders * kLoaders;
  while (n > 0 && (2 * n) % kComputeWarps) n -= kLoaders;
  return n < 2 * kLoaders ? 0 : n;
}

namespace {
struct SpecEntry {
  int rh, ro, rd, g, dpl;
  const void *(*kernel)();          // one sequence per instruction
  const void *(*kernel_batched)();  // up to kMaxBatch sequences (or null)
  const void *(*kernel_batched_tqo)();  // the same with tensor-core QKV / O (or null)
};
// Shapes with a specialised build: Llama-3.2-1B (hidden 2048, 32/8 heads of
// 64; also batched) and Llama-3.1-8B (hidden 4096, 32/8 heads of 128).
const SpecEntry kSpecs[] = {
    {4, 4, 4, 4, 2, spec_kernel_llama1b, spec_kernel_llama1b_batched, spec_kernel_llama1b_batched_tqo},
    {2, 2, 4, 4, 4, spec_kernel_llama8b, nullptr, nullptr},
};
}  // namespace

const void *interp_kernel_for(const KParams &p, bool specialised, int nb, bool tqo, int *variant) {
  if (variant) *variant = 0;
  if (specialised && p.nkv > 0) {
    const int g = p.nq / p.nkv, dpl = p.d / 32;
    for (const SpecEntry &e : kSpecs)
      if (e.rh == p.Rh && e.ro == p.Ro && e.rd == p.Rd && e.g == g && e.dpl == dpl) {
        const auto batched = tqo ? e.kernel_batched_tqo : e.kernel_batched;
        if (nb > 1 && !batched) return nullptr;
        if (variant) *variant = 1;
        return nb > 1 ? batched() : e.kernel();
      }
  }
  if (nb > 1) return nullptr;
  return (const void *)interp_kernel<1, false, SpecGeneric>;
}

const void *interp_kernel_raw() { return (const void *)interp_kernel<1, true, SpecGeneric>; }

const void *interp_kernel_tp() { return (const void *)interp_kernel<1, false, SpecGenericTP>; }

cudaError_t interp_prepare(const void *fn, int smem, int *blocks_per_sm) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fn, kThreads, smem);
}

cudaError_t launch_interp(const void *fn, const KParams &p, int grid, int smem, cudaStream_t st, bool cooperative) {
  void *args[] = {const_cast<KParams *>(&p)};
  if (cooperative) return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), args, (size_t)smem, st);
  return cudaLaunchKernel(fn, dim3(grid), dim3(kThreads), args, (size_t)smem, st);
}

}  // namespace mk
