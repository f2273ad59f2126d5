// moe_align: group the T*k (token, slot) assignments by expert, bit-exact
// (the device body and its output contract are in align_cta.cuh).  One CTA
// (at least E threads; more warps for large T*k), or, from T*k = 8192 on, two
// grids over slices of the flat index range.
#include <cuda_runtime.h>

#include "align_cta.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(1024) align_kernel(AlignArgs a, int mode, int slice) {
  extern __shared__ int sh[];
  pdl_wait();
  pdl_launch_next();
  align_cta(a, mode, slice, sh);
}

cudaError_t launch_align(const AlignArgs& a, cudaStream_t st) {
  const long long A = static_cast<long long>(a.T) * a.k;
  const int e32 = (a.E + 31) / 32 * 32;
  auto kern = align_kernel;
  if (A < kAlignSliceMin || a.slice_hist == nullptr) {
    // one CTA: 8 warps suffice for decode-sized T*k, 32 shorten the
    // per-warp walks of mid-sized batches
    int threads = A >= 8192 ? 1024 : 256;
    if (threads < e32) threads = e32;
    const size_t smem = static_cast<size_t>(threads / 32) * a.E * sizeof(int);
    cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(kern, dim3(1), dim3(threads), smem, st, a, 0, 0);
  }
  // two grids over slices of >= kAlignSliceMin / 8 assignments, at most kAlignMaxSlices
  long long nb = (A + kAlignSliceMin / 8 - 1) / (kAlignSliceMin / 8);
  if (nb > kAlignMaxSlices) nb = kAlignMaxSlices;
  const int slice = static_cast<int>((A + nb - 1) / nb);
  int threads = 256;
  if (threads < e32) threads = e32;
  const size_t smem = static_cast<size_t>(threads / 32) * a.E * sizeof(int);
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = launch_pdl(kern, dim3(static_cast<int>(nb)), dim3(threads), smem, st, a, 1, slice);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(static_cast<int>(nb)), dim3(threads), smem, st, a, 2, slice);
}

}  // namespace moe
