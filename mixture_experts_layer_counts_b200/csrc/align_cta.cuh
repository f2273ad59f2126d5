// Device body of moe_align (one CTA's part of it).
//
// Output contract (unpadded): counts[e]; offsets = exclusive prefix sum of
// counts (E+1 entries); perm[p] = flat index f = t*k + j of the p-th
// assignment in expert-major order, ascending f inside an expert (a stable
// counting sort); inv_perm[perm[p]] = p.  The same pass builds the tile
// schedule of the grouped GEMMs (token chunks per expert, per orientation)
// and, on the FP8 path, the per-tensor activation scale s1 = amax|x| / 448.
//
// Each warp owns a contiguous slice of the flat indices; a per-warp histogram
// (lanes with equal experts found by ballots on the id bits, the lowest such
// lane adds the group size) gives every warp its starting position per
// expert, so the scatter is stable without atomics.
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ int block_exclusive_scan(int v, int* tmp32, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) tmp32[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? tmp32[lane] : 0;
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += o;
    }
    tmp32[lane] = wi - w;   // exclusive warp offsets
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = tmp32[warp] + incl - v;
  __syncthreads();
  return r;
}

// Mask of the warp's lanes holding the same key (0 <= key < 2^nbits): one
// ballot per key bit (cheaper than a match instruction on many distinct keys).
__device__ __forceinline__ unsigned same_key_lanes(int key, int nbits) {
  unsigned m = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

}  // namespace

// mode 0: the whole job in one CTA.  Large T*k runs as two grids over
// slices of the flat index range, one slice per CTA: mode 1 writes each
// CTA's per-expert counts to a.slice_hist; mode 2 recomputes its own slice's
// per-warp counts, places the slice after the earlier slices' assignments of
// each expert (prefix over slice_hist) and scatters; its CTA 0 also writes
// counts, offsets, the tile schedule and the FP8 scale.
__device__ __forceinline__ void align_cta(const AlignArgs& a, int mode, int slice, int* hist) {
  // blockDim.x: a multiple of 32, >= E, <= 1024; hist: [warps][E] ints of shared memory
  __shared__ int tmp32[32];
  __shared__ int total;
  __shared__ float famax[32];
  const int E = a.E;
  const int A = a.T * a.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int NW = blockDim.x >> 5;
  const int cbeg = mode == 0 ? 0 : min(A, static_cast<int>(blockIdx.x) * slice);
  const int cend = mode == 0 ? A : min(A, cbeg + slice);
  const bool lead = mode == 0 || (mode == 2 && blockIdx.x == 0);   // writes the shared outputs

  // FP8 activation scale inputs, requested now so they arrive during the histogram
  float m_pre = 0.f;
  if (lead && a.amax_tok != nullptr)
    for (int t = threadIdx.x; t < a.T; t += blockDim.x) m_pre = fmaxf(m_pre, __ldcg(a.amax_tok + t));
  for (int i = threadIdx.x; i < NW * E; i += blockDim.x) hist[i] = 0;
  if (a.gemm_flags != nullptr && (mode == 0 || (mode == 1 && blockIdx.x == 0)))
    for (int i = threadIdx.x; i < a.n_gemm_flags; i += blockDim.x) a.gemm_flags[i] = 0;
  __syncthreads();

  // each warp walks its part of the slice in ascending flat index, kBatch
  // loads of 32 ids in flight at a time
  constexpr int kBatch = 8;
  const int kbits = 32 - __clz(E);   // bits of the keys 0..E (E = "no expert")
  const int per = (cend - cbeg + NW - 1) / NW;
  const int beg = min(cend, cbeg + warp * per), end = min(cend, beg + per);
  // a slice of at most one batch per warp (decode-sized calls) keeps its ids
  // in registers for the scatter pass instead of loading them again
  const bool one_batch = per <= 32 * kBatch;
  int keep[kBatch];
  for (int base = beg; base < end; base += 32 * kBatch) {
    int ev[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int f = base + 32 * u + lane;
      ev[u] = f < end ? __ldcg(a.topk_ids + f) : -1;
      keep[u] = ev[u];
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (base + 32 * u >= end) break;   // warp-uniform
      int e = ev[u];
      if (e >= E || e < -1) {
        if (mode != 2) report_status(a.hdr, MOE_DEVICE_BOUNDS, 0x100u);
        e = -1;
      }
      const unsigned grp = same_key_lanes(e < 0 ? E : e, kbits);
      if (e >= 0 && lane == __ffs(grp) - 1) hist[warp * E + e] += __popc(grp);
      __syncwarp();
    }
  }
  __syncthreads();

  if (mode == 1) {   // slice totals per expert
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int c = 0;
      for (int w = 0; w < NW; ++w) c += hist[w * E + e];
      a.slice_hist[static_cast<size_t>(blockIdx.x) * E + e] = c;
    }
    return;
  }

  // counts, offsets, per-warp starting positions
  int c = 0, before = 0;   // count of expert threadIdx.x; its assignments in earlier slices
  if (threadIdx.x < E) {
    if (mode == 0) {
      for (int w = 0; w < NW; ++w) c += hist[w * E + threadIdx.x];
    } else {
      for (int b = 0; b < static_cast<int>(gridDim.x); ++b) {
        const int h = a.slice_hist[static_cast<size_t>(b) * E + threadIdx.x];
        if (b < static_cast<int>(blockIdx.x)) before += h;
        c += h;
      }
    }
  }
  const int excl = block_exclusive_scan(threadIdx.x < E ? c : 0, tmp32, &total);
  if (threadIdx.x < E) {
    if (lead) {
      a.counts[threadIdx.x] = c;
      a.offsets[threadIdx.x] = excl;
    }
    int run = excl + before;
    for (int w = 0; w < NW; ++w) {
      const int h = hist[w * E + threadIdx.x];
      hist[w * E + threadIdx.x] = run;
      run += h;
    }
  }
  if (threadIdx.x == 0 && lead) a.offsets[E] = total;
  __syncthreads();

  // stable scatter
  for (int base = beg; base < end; base += 32 * kBatch) {
    int ev[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int f = base + 32 * u + lane;
      ev[u] = one_batch ? keep[u] : (f < end ? __ldcg(a.topk_ids + f) : -1);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (base + 32 * u >= end) break;   // warp-uniform
      const int f = base + 32 * u + lane;
      int e = ev[u];
      if (e >= E || e < -1) e = -1;
      const unsigned grp = same_key_lanes(e < 0 ? E : e, kbits);
      const int rank = __popc(grp & ((1u << lane) - 1u));
      if (e >= 0) {
        const int pos = hist[warp * E + e] + rank;
        a.perm[pos] = f;
        a.inv_perm[f] = pos;
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(grp) - 1) hist[warp * E + e] += __popc(grp);
      __syncwarp();
    }
  }
  if (!lead) return;

  // tile schedule: swap-AB chunks of <= swap_chunk tokens for experts
  // with count <= swap_max_count, normal-orientation tiles of kNormalTokens
  // tokens (down GEMM) and of kPairTokens tokens (gate/up GEMM) for the rest.
  const bool ex = threadIdx.x < E && c > 0;
  const bool sw = ex && c <= a.swap_max_count;
  const int nsw = sw ? (c + a.swap_chunk - 1) / a.swap_chunk : 0;
  const int nno = (ex && !sw) ? (c + kNormalTokens - 1) / kNormalTokens : 0;
  const int osw = block_exclusive_scan(nsw, tmp32, &total);
  const int tsw = total;
  __syncthreads();
  const int ono = block_exclusive_scan(nno, tmp32, &total);
  const int tno = total;
  __syncthreads();
  const int npr = (ex && !sw) ? (c + kPairTokens - 1) / kPairTokens : 0;
  const int opr = block_exclusive_scan(npr, tmp32, &total);
  const int tpr = total;
  for (int i = 0; i < nsw; ++i) {
    const int n0 = i * a.swap_chunk;
    a.chunks_swap[osw + i] = make_int4(threadIdx.x, excl + n0, min(a.swap_chunk, c - n0), i);
  }
  for (int i = 0; i < nno; ++i) {
    const int n0 = i * kNormalTokens;
    a.chunks_normal[ono + i] = make_int4(threadIdx.x, excl + n0, min(kNormalTokens, c - n0), i);
  }
  for (int i = 0; i < npr; ++i) {
    const int n0 = i * kPairTokens;
    a.chunks_pair[opr + i] = make_int4(threadIdx.x, excl + n0, min(kPairTokens, c - n0), i);
  }
  if (threadIdx.x == 0) {
    a.hdr[kHdrChunksSwap] = static_cast<uint32_t>(tsw);
    a.hdr[kHdrChunksNormal] = static_cast<uint32_t>(tno);
    a.hdr[kHdrChunksPair] = static_cast<uint32_t>(tpr);
    a.hdr[kHdrBarrier] = 0u;   // arrival counter of the gate/up GEMM's closing grid barrier
  }

  // FP8 activation scale: s1 = amax / 448 (one IEEE fp32 division); amax == 0 -> 1
  if (a.amax_tok != nullptr) {
    float m = m_pre;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (lane == 0) famax[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float mm = 0.f;
      for (int w = 0; w < NW; ++w) mm = fmaxf(mm, famax[w]);
      const float s1 = mm == 0.f ? 1.0f : __fdiv_rn(mm, 448.0f);
      a.hdr[kHdrScaleS1] = __float_as_uint(s1);
    }
  }
}

}  // namespace moe
