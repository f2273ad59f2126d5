// Device helpers shared by the grouped GEMM kernels (gemm.cu) and the fused
// swap-AB expert FFN kernel (ffn.cu): the stream-K work split, the unit ->
// tile mapping, bounded flag waits and the FP8 requantisation tail.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

constexpr int kMinAtomsPerCta = 8;   // below this, fewer CTAs share the work

// Contiguous atom range of CTA c out of G over W atoms, and the CTA owning atom a.
__device__ __forceinline__ long long range_begin(long long W, int G, int c) {
  return static_cast<long long>(c) * W / G;
}
__device__ __forceinline__ int atom_owner(long long a, long long W, int G) {
  return static_cast<int>(((a + 1) * G - 1) / W);
}

// Walks one CTA's work as (unit, first atom, end atom) segments: either a
// contiguous atom range [a, a1) (balanced split), or (rr) whole units
// u_next, u_next + step, ... < u_end dealt round-robin.
struct Segments {
  long long a, a1;
  int katoms;
  bool rr;
  long long u_next, u_end;
  int step;
  __device__ bool next(int& u, int& kb0, int& kb1) {
    if (rr) {
      if (u_next >= u_end) return false;
      u = static_cast<int>(u_next);
      kb0 = 0;
      kb1 = katoms;
      u_next += step;
      return true;
    }
    if (a >= a1) return false;
    u = static_cast<int>(a / katoms);
    kb0 = static_cast<int>(a - static_cast<long long>(u) * katoms);
    const long long left = a1 - a;
    kb1 = left < katoms - kb0 ? kb0 + static_cast<int>(left) : katoms;
    a += kb1 - kb0;
    return true;
  }
};

// Unit -> (token chunk, weight tile).  Swap-AB: chunk-major.  Normal
// orientation: inside one expert, weight tile major and token chunk minor, so
// the token chunks that share a weight tile are consecutive units; dealt
// round-robin, they run on neighbouring CTAs at the same time and share one
// DRAM fetch of that tile through L2.  chunk.w = index of the chunk inside its
// expert; the expert has ceil(counts[e] / kChunkTokens) chunks.
template <bool kGrouped, int kChunkTokens>
__device__ __forceinline__ void unit_coords(const GemmArgs& a, int u, int4& ch, int& mt) {
  const int cs = u / a.mtiles;   // a chunk of the unit's expert
  if constexpr (!kGrouped) {
    if (a.dense_T > 0) {   // router logits: dense chunks of dense_chunk hidden rows
      mt = u - cs * a.mtiles;
      const int n0 = cs * a.dense_chunk;
      ch = make_int4(0, n0, min(a.dense_chunk, a.dense_T - n0), cs);
      return;
    }
    ch = a.chunks[cs];
    mt = u - cs * a.mtiles;
  } else {
    const int4 s = a.chunks[cs];
    const int c0 = cs - s.w;   // the expert's first chunk
    const int nch = (a.counts[s.x] + kChunkTokens - 1) / kChunkTokens;
    const int local = u - c0 * a.mtiles;
    mt = local / nch;
    ch = a.chunks[c0 + (local - mt * nch)];
  }
}

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <int kEpiThreads>
__device__ __forceinline__ void epilogue_bar() {   // the epilogue warps only
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for a neighbour CTA's partial-tile flag.
__device__ __forceinline__ bool wait_flag(const int* flag, volatile int* abort, uint32_t* status,
                                          unsigned long long timeout_ns) {
  if (ld_acquire(flag) != 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire(flag) != 0) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        report_status(status, MOE_DEVICE_TIMEOUT, kSiteGridBarrier);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Closing step of the last FP8 gate/up launch of a call: the per-tensor
// requantisation of the intermediate.  Every CTA of the grid arrives at a
// grid barrier once its epilogue stores and its amax|h| slot are written
// (fence, then an integer arrival count); then each CTA forms
// s2 = max(amax slots) / 448 (one IEEE fp32 division; amax 0 gives 1) and
// writes E4M3(h / s2), round-to-nearest-even and saturating to +-448, for a
// grid-strided part of the intermediate.  The wait is bounded: on expiry the
// status word records it and the CTA returns without requantising.
__device__ __forceinline__ void requant_tail(const GemmArgs& a, float* s_s2, volatile int* s_ok) {
  __threadfence();   // this thread's stores of h (and amax) are visible device-wide
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(a.hdr + kHdrBarrier, 1u);
    const unsigned int need = gridDim.x;
    bool ok = true;
    if (ld_acquire(reinterpret_cast<const int*>(a.hdr + kHdrBarrier)) < static_cast<int>(need)) {
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t it = 1;; ++it) {
        if (ld_acquire(reinterpret_cast<const int*>(a.hdr + kHdrBarrier)) >= static_cast<int>(need)) break;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > a.timeout_ns) {
          report_status(a.hdr, MOE_DEVICE_TIMEOUT, kSiteGridBarrier);
          ok = false;
          break;
        }
      }
    }
    float m = 0.f;
    for (int i = 0; ok && i < a.amax_n; ++i) m = fmaxf(m, __ldcg(a.amax_all + i));
    const float s2 = m == 0.f ? 1.0f : __fdiv_rn(m, 448.0f);
    if (ok && blockIdx.x == 0) a.hdr[kHdrScaleS2] = __float_as_uint(s2);
    *s_s2 = s2;
    *s_ok = ok ? 1 : 0;
  }
  __syncthreads();
  if (!*s_ok) return;
  const float s2 = *s_s2;
  const float4* h = static_cast<const float4*>(a.out);
  uint32_t* q = static_cast<uint32_t*>(a.inter_q);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  constexpr int kU = 8;   // loads in flight per thread
  for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < a.requant_n4;
       i0 += kU * stride) {
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i0 + u * stride < a.requant_n4) v[u] = __ldcg(h + i0 + u * stride);
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i0 + u * stride < a.requant_n4)
        q[i0 + u * stride] = pack_e4m3x4(__fdiv_rn(v[u].x, s2), __fdiv_rn(v[u].y, s2), __fdiv_rn(v[u].z, s2),
                                         __fdiv_rn(v[u].w, s2));
  }
}

}  // namespace moe
