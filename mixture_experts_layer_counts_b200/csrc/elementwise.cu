// Bandwidth-bound helper kernels of the layer:
//   gather   x_perm[p] = hidden[perm[p] / k]  (bf16), or its per-tensor E4M3
//            quantisation x / s1 (FP8 path; one IEEE fp32 division, RNE,
//            saturating to +-448)
//   combine  out[t] = bf16(sum_{j<k} ysc[t*k + j]) in slot order, fp32 sum
//            (calls with normal-orientation experts; otherwise the down GEMM's
//            epilogue combines)
// All grids are sized from the SM count; 16-byte vector accesses.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {
int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}
}  // namespace

// Work unit = (row p, block of 256 16-byte columns); a CTA takes kU units
// per iteration so their perm and row loads are in flight together, and no
// per-element integer division is needed.
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ hidden,
                                                     const int32_t* __restrict__ perm, int A, int k,
                                                     int vpr, uint4* __restrict__ xperm) {
  pdl_wait();
  pdl_launch_next();
  const int T = A / k;
  const int nb = (vpr + 255) / 256;   // column blocks per row
  const int units = A * nb;
  constexpr int kU = 4;
  for (int u0 = blockIdx.x; u0 < units; u0 += kU * gridDim.x) {
    int t[kU], p[kU], col[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int unit = min(u0 + u * static_cast<int>(gridDim.x), units - 1);
      p[u] = unit / nb;
      col[u] = (unit - p[u] * nb) * 256 + threadIdx.x;
      t[u] = min(max(perm[p[u]] / k, 0), T - 1);   // perm is a bijection; clamp is a guard
    }
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (col[u] < vpr) v[u] = hidden[static_cast<size_t>(t[u]) * vpr + col[u]];
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (u0 + u * static_cast<int>(gridDim.x) < units && col[u] < vpr)
        xperm[static_cast<size_t>(p[u]) * vpr + col[u]] = v[u];
  }
}

__global__ void gather_quant_kernel(const uint4* __restrict__ hidden, const int32_t* __restrict__ perm,
                                    int A, int k, int vpr, const uint32_t* __restrict__ hdr,
                                    uint2* __restrict__ xq) {
  pdl_wait();
  pdl_launch_next();
  const int T = A / k;
  const float s1 = __uint_as_float(hdr[kHdrScaleS1]);
  const size_t n = static_cast<size_t>(A) * vpr;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / vpr);
    const int c = static_cast<int>(i - static_cast<size_t>(p) * vpr);
    const int t = min(max(perm[p] / k, 0), T - 1);   // perm is a bijection; clamp is a guard
    const uint4 v = hidden[static_cast<size_t>(t) * vpr + c];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 q = __bfloat1622float2(b[j]);
      f[2 * j] = __fdiv_rn(q.x, s1);
      f[2 * j + 1] = __fdiv_rn(q.y, s1);
    }
    xq[i] = make_uint2(pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]));
  }
}

// Combine pass (used when some experts run in the normal orientation):
// out[t] = sum_{j<k} ysc[t*k + j] in slot order, fp32, then one bf16 rounding
// (or the unrounded fp32 sum for a tensor-parallel partial).  Work unit =
// (token t, block of 256 float4 columns); per thread the k slot loads are
// issued together and summed in slot order.
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ ysc, int T, int k,
                                                      int h4, void* __restrict__ out, int out_f32) {
  pdl_wait();
  pdl_launch_next();
  const int nb = (h4 + 255) / 256;
  const int units = T * nb;
  for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const int t = unit / nb;
    const int c = (unit - t * nb) * 256 + threadIdx.x;
    if (c >= h4) continue;
    const float4* src = ysc + static_cast<size_t>(t) * k * h4 + c;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += 8) {
      float4 y[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u < k) y[u] = __ldcg(src + static_cast<size_t>(j0 + u) * h4);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (j0 + u < k) {
          if (j0 + u == 0) {
            acc = y[u];
          } else {
            acc.x += y[u].x;
            acc.y += y[u].y;
            acc.z += y[u].z;
            acc.w += y[u].w;
          }
        }
      }
    }
    if (out_f32) {
      static_cast<float4*>(out)[static_cast<size_t>(t) * h4 + c] = acc;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      static_cast<uint2*>(out)[static_cast<size_t>(t) * h4 + c] =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

cudaError_t launch_combine(const float* ysc, int T, int k, int H, void* out, bool out_f32, cudaStream_t st) {
  const int h4 = H / 4;
  const int units = T * ((h4 + 255) / 256);
  const int grid = std::min(units, sm_count() * 8);
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, st, reinterpret_cast<const float4*>(ysc), T, k,
                    h4, out, out_f32 ? 1 : 0);
}

// Tensor-parallel sum: out[i] = bf16(parts[0][i] + parts[1][i] + ... ), the
// partials added in rank order from the first, one rounding at the end.
__global__ void __launch_bounds__(256) sum_partials_kernel(const float4* __restrict__ parts, int G,
                                                           long long n4, uint2* __restrict__ out) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 acc = parts[i];
    for (int g = 1; g < G; ++g) {
      const float4 v = parts[static_cast<long long>(g) * n4 + i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    out[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
  }
}

cudaError_t launch_sum_partials(const float* parts, int G, long long n, __nv_bfloat16* out, cudaStream_t st) {
  const long long n4 = n / 4;
  const int grid = static_cast<int>(std::min<long long>((n4 + 255) / 256, static_cast<long long>(sm_count()) * 8));
  sum_partials_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(reinterpret_cast<const float4*>(parts), G, n4,
                                                          reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

// Debug output: dst[t] = src[inv_perm[t * k]] (the first slot's copy of a
// token row in perm order back in token order), 16-byte vectors.
__global__ void unpermute_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ inv_perm,
                                      int T, int k, int vpr, uint4* __restrict__ dst) {
  const size_t n = static_cast<size_t>(T) * vpr;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vpr);
    const int c = static_cast<int>(i - static_cast<size_t>(t) * vpr);
    const int p = inv_perm[static_cast<size_t>(t) * k];
    if (p >= 0 && p < T * k) dst[i] = src[static_cast<size_t>(p) * vpr + c];
  }
}

cudaError_t launch_unpermute_rows(const void* src, const int32_t* inv_perm, int T, int k, int row_bytes,
                                  void* dst, cudaStream_t st) {
  const int vpr = row_bytes / 16;
  const size_t n = static_cast<size_t>(T) * vpr;
  const int grid = static_cast<int>(std::min<size_t>((n + 255) / 256, static_cast<size_t>(sm_count()) * 4));
  unpermute_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(src), inv_perm, T, k, vpr,
                                              static_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_gather(const __nv_bfloat16* hidden, const int32_t* perm, int A, int k, int H,
                          bool fp8, const uint32_t* hdr, void* xperm, cudaStream_t st) {
  const int vpr = H / 8;
  const size_t n = static_cast<size_t>(A) * vpr;
  const int grid = static_cast<int>(std::min<size_t>((n + 255) / 256, static_cast<size_t>(sm_count()) * 8));
  const int units = A * ((vpr + 255) / 256);
  const int ggrid = std::min(units, sm_count() * 8);
  if (fp8)
    return launch_pdl(gather_quant_kernel, dim3(grid), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(hidden), perm, A, k, vpr, hdr,
                      reinterpret_cast<uint2*>(xperm));
  return launch_pdl(gather_kernel, dim3(ggrid), dim3(256), 0, st, reinterpret_cast<const uint4*>(hidden),
                    perm, A, k, vpr, reinterpret_cast<uint4*>(xperm));
}

}  // namespace moe
