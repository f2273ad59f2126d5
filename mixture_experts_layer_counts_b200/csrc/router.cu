// Router: logits, fp32 softmax, top-k (ties -> lower expert index),
// renormalisation.
//
// The selection is defined on the exact real-valued logits of the bf16 inputs
// (the pages give no precision for routing; exactness makes "bit-exact
// routing" independent of summation order).  Three tiers:
//   1. fp32 logits with a rigorous error bound.  Products of two bf16 values
//      are exact in fp32, so each logit carries only summation error,
//      |err| <= gamma_n * sum|x*w| <= gamma_n * ||x|| * ||w|| (n = the
//      longest chain of roundings of the logit kernel that ran: H/32
//      sequential FMAs per lane plus the 5-level warp butterfly, or 64-term
//      blocks summed in sequence for the tiled large-batch kernel), plus one
//      rounding for the bias.
//   2. A token whose top-(k+1) ordering is not separated by twice that bound
//      re-evaluates only its candidate experts in fp64 (bound ~1e-16 rel).
//   3. Candidates still within 2x the fp64 bound of each other are ordered by
//      their exact values, accumulated as 640-bit fixed-point integers.
// Softmax and the renormalised weights are computed in fp32 from the fp32
// logits, one warp per token with shuffle reductions.
// Large batches take their logits from the tensor cores instead (a dense
// swap-AB GEMM of the grouped-GEMM kernel).  Their bound is loose (the
// accumulation order and rounding inside the MMA are not specified), so every
// token goes through tier 2 for its candidates, first in mixed precision (fp32
// blocks of 8 products, fp64 sums: a bound of about 7 fp32 ulps of sum|x w|),
// then in fp64 when that leaves a gap open; the weights come from those
// re-evaluated logits.
#include <cuda_bf16.h>

#include <cfloat>
#include <cstdlib>

#include "align_cta.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kLimbs = 20;      // 20 x 32-bit limbs: bit b <-> 2^(b - kExactOffset)
constexpr int kExactOffset = 300;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// (value desc, index asc) total order used for top-k.
__device__ __forceinline__ bool beats(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// ---- exact fixed-point accumulation of bf16 products (tier 3) -------------
// A bf16 value is sign * m * 2^q with m an 8-bit integer (hidden bit
// included) and q = exponent_field - 134 (normal) or -133 (subnormal).
__device__ __forceinline__ void bf16_parts(uint16_t b, uint32_t& m, int& q, uint32_t& s) {
  s = b >> 15;
  const uint32_t ef = (b >> 7) & 0xFFu;
  const uint32_t f = b & 0x7Fu;
  if (ef == 0) {
    m = f;
    q = -133;
  } else {
    m = f | 0x80u;
    q = static_cast<int>(ef) - 134;
  }
}

__device__ __forceinline__ void limb_add(long long (&acc)[kLimbs], uint64_t mag, int bitpos,
                                         bool neg) {
  const int li = bitpos >> 5;
  const uint64_t v = mag << (bitpos & 31);   // mag < 2^24, shift < 32: fits 64 bits
  const long long lo = static_cast<long long>(v & 0xFFFFFFFFull);
  const long long hi = static_cast<long long>(v >> 32);
  if (neg) {
    acc[li] -= lo;
    acc[li + 1] -= hi;
  } else {
    acc[li] += lo;
    acc[li + 1] += hi;
  }
}

// Exact logit of (token row x, expert row w) + bias, normalised limbs, in
// every lane of the warp.
__device__ void exact_logit(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w,
                            float bias, int H, long long (&acc)[kLimbs]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) acc[i] = 0;
  for (int h = lane; h < H; h += 32) {
    uint32_t mx, mw, sx, sw;
    int qx, qw;
    bf16_parts(x[h], mx, qx, sx);
    bf16_parts(w[h], mw, qw, sw);
    if (mx == 0 || mw == 0) continue;
    limb_add(acc, static_cast<uint64_t>(mx) * mw, qx + qw + kExactOffset, (sx ^ sw) != 0);
  }
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) acc[i] = warp_sum_ll(acc[i]);
  if (bias != 0.0f) {
    const uint32_t b = __float_as_uint(bias);
    const uint32_t ef = (b >> 23) & 0xFFu;
    const uint32_t f = b & 0x7FFFFFu;
    const uint32_t m = ef == 0 ? f : (f | 0x800000u);
    const int q = ef == 0 ? -149 : static_cast<int>(ef) - 150;
    limb_add(acc, m, q + kExactOffset, (b >> 31) != 0);
  }
  // carry-normalise: limbs 0..18 in [0, 2^32), the top limb keeps the sign
#pragma unroll
  for (int i = 0; i < kLimbs - 1; ++i) {
    const long long c = acc[i] >> 32;   // arithmetic shift = floor division
    acc[i] -= c * 4294967296LL;
    acc[i + 1] += c;
  }
}

__device__ __forceinline__ int exact_cmp(const long long (&a)[kLimbs], const long long (&b)[kLimbs]) {
#pragma unroll
  for (int i = kLimbs - 1; i >= 0; --i) {
    if (a[i] != b[i]) return a[i] > b[i] ? 1 : -1;
  }
  return 0;
}

// Up to four logits of one token row at once (tier 2): the warp walks the
// row once, each lane loading its 16-byte piece of x and of every router row
// (two pieces of each in flight), exact products accumulated with one
// accumulator per row and per half of the unrolled pair, then the butterfly.
// kMixed = false: every product added in fp64; each term passes through at
// most H/32 + 6 roundings, inside the H/32 + 16 of the fp64 bound.
// kMixed = true: the 8 products of each 16-byte vector pair summed by an fp32
// FMA chain (7 roundings), the vector sums added in fp64: one fp64
// conversion per 8 products instead of two per product; error at most
// (7 u32 + (H/256 + 16) u64) sum|x w| (1 + 1e-4), plus H 2^-148 for values
// below fp32's normal range.
template <bool kMixed>
__device__ void logits4(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* const (&w)[4], int nw,
                        int H, double (&out)[4]) {
  const int lane = threadIdx.x & 31;
  const int vpr = H / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  double acc[4][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
  for (int c0 = lane; c0 < vpr; c0 += 64) {
    uint4 xs[2], ws[4][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = c0 + 32 * u;
      xs[u] = c < vpr ? xv[c] : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int r = 0; r < 4; ++r)
        ws[r][u] = (r < nw && c < vpr) ? reinterpret_cast<const uint4*>(w[r])[c] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float xf[8];
      unpack8(xs[u], xf);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float wf[8];
        unpack8(ws[r][u], wf);
        if constexpr (kMixed) {
          float p = xf[0] * wf[0];
#pragma unroll
          for (int i = 1; i < 8; ++i) p = fmaf(xf[i], wf[i], p);
          acc[r][u] += static_cast<double>(p);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[r][u] = fma(static_cast<double>(xf[i]), static_cast<double>(wf[i]), acc[r][u]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) out[r] = warp_sum_d(acc[r][0] + acc[r][1]);
}

// Rank the nc candidates (c_idx, c_val) by (value desc, index asc) into
// c_ord (c_ord[rank] = candidate slot), by the calling warp.
__device__ void rank_candidates(const int* c_idx, int* c_ord, const double* c_val, int nc) {
  const int lane = threadIdx.x & 31;
  for (int c = lane; c < nc; c += 32) c_ord[c] = c;   // valid even if ranks collide (NaN)
  __syncwarp();
  for (int c = lane; c < nc; c += 32) {
    const double vc = c_val[c];
    const int ic = c_idx[c];
    int rank = 0;
    for (int j = 0; j < nc; ++j) {
      const double vj = c_val[j];
      rank += (vj > vc || (vj == vc && c_idx[j] < ic)) ? 1 : 0;
    }
    if (rank < nc) c_ord[rank] = c;
  }
  __syncwarp();
}

// The k selected experts in order, from ranked candidates whose values carry
// errors below margin / 2 (by the calling warp).  Runs of candidates closer
// than `margin` are ordered by their exact values (tier 3); put(e, d) takes
// them in order.  Marks chosen candidates with c_idx = -1.
template <typename Put>
__device__ void assemble_in_order(int* c_idx, const int* c_ord, const double* c_val, int nc, int k,
                                  double margin, const __nv_bfloat16* __restrict__ xrow,
                                  const __nv_bfloat16* __restrict__ router_w, const float* __restrict__ bias,
                                  int H, int& got, Put&& put) {
  const int lane = threadIdx.x & 31;
  int pos = 0;
  const uint16_t* xbits = reinterpret_cast<const uint16_t*>(xrow);
  while (got < k && pos < nc) {
    int end = pos;
    while (end + 1 < nc && !(c_val[c_ord[end]] - c_val[c_ord[end + 1]] > margin)) ++end;
    if (end == pos) {
      put(c_idx[c_ord[pos]], c_val[c_ord[pos]]);
      pos = end + 1;
      continue;
    }
    const int need = min(end - pos + 1, k - got);
    for (int q = 0; q < need; ++q) {
      long long best[kLimbs];
      int best_e = -1, best_slot = -1;
      for (int m = pos; m <= end; ++m) {
        const int e = c_idx[c_ord[m]];
        if (e < 0) continue;   // already chosen
        long long cur[kLimbs];
        exact_logit(xbits, reinterpret_cast<const uint16_t*>(router_w) + static_cast<size_t>(e) * H,
                    bias ? bias[e] : 0.f, H, cur);
        int cmp = best_e < 0 ? 1 : exact_cmp(cur, best);
        if (cmp > 0 || (cmp == 0 && e < best_e)) {
#pragma unroll
          for (int i = 0; i < kLimbs; ++i) best[i] = cur[i];
          best_e = e;
          best_slot = m;
        }
      }
      put(best_e, c_val[c_ord[best_slot]]);
      __syncwarp();
      if (lane == 0) c_idx[c_ord[best_slot]] = -1;
      __syncwarp();
    }
    pos = end + 1;
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Kernel 1: logits[t, e] = sum_h x[t,h] w[e,h] + b[e], stored as fp32.
// ACC = kAcc64: every product accumulated in fp64 (the smallest decode
// calls; the bound is then the fp64 chain plus the final fp32 rounding).
// ACC = kAccMixed: the 8 exact products of each 16-byte vector pair are summed
// by an fp32 FMA chain (7 roundings) and the vector sums accumulated in fp64,
// one fp64 conversion per 8 products instead of two per product (larger
// decode calls, where conversions would dominate); bound 7 fp32 ulps of
// sum|x w| plus the fp64 chain.  ACC = kAcc32: plain fp32 chains.  Plus ||x_t||,
// ||w_e|| for the error bound and per-token amax|x| for the FP8 activation
// scale.  CTA = TT tokens x 8 experts (one expert per warp), hidden rows
// staged in smem, four 16-byte router-row loads in flight per lane.
// ---------------------------------------------------------------------------
constexpr int kAcc32 = 0, kAcc64 = 1, kAccMixed = 2;

// The CTA body (warps 0..7 compute; any further warps only help staging).
template <int TT, int ACC>
__device__ __forceinline__ void logits_body(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ router_w,
    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits,
    float* __restrict__ xnorm, float* __restrict__ wnorm, float* __restrict__ amax_tok, uint4* sx,
    bool every_cta_wnorm = false) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int t0 = blockIdx.x * TT;
  const int nt = min(TT, T - t0);
  const int vpr = H / 8;   // 16-byte vectors per row
  const uint4* hv = reinterpret_cast<const uint4*>(hidden);
  const int e = blockIdx.y * 8 + warp;
  const bool has_e = warp < 8 && e < E;
  const uint4* wrow = reinterpret_cast<const uint4*>(router_w) + static_cast<size_t>(has_e ? e : 0) * vpr;
  constexpr int U = 8;     // 16-byte router-row loads in flight per lane

  // the first U vectors of this warp's router row are requested before the
  // token rows are staged, so both sets of loads are in flight together
  uint4 wv[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = lane + 32 * u;
    wv[u] = (has_e && c < vpr) ? wrow[c] : make_uint4(0, 0, 0, 0);
  }
  for (int i0 = threadIdx.x; i0 < TT * vpr; i0 += 4 * blockDim.x) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      const int r = i / vpr;
      v[u] = (i < TT * vpr && r < nt) ? hv[static_cast<size_t>(t0 + r) * vpr + (i - r * vpr)]
                                      : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < TT * vpr) sx[i] = v[u];
    }
  }
  __syncthreads();

  if (blockIdx.y == 0) {
    for (int r = warp; r < nt; r += nwarps) {
      float ss = 0.f, am = 0.f;
      for (int c = lane; c < vpr; c += 32) {
        float f[8];
        unpack8(sx[r * vpr + c], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ss = fmaf(f[i], f[i], ss);
          am = fmaxf(am, fabsf(f[i]));
        }
      }
      ss = warp_sum(ss);
      am = warp_max(am);
      if (lane == 0) {
        xnorm[t0 + r] = sqrtf(ss);
        amax_tok[t0 + r] = am;
      }
    }
  }

  if (!has_e) return;
  constexpr bool F64 = ACC != kAcc32;
  using Acc = typename std::conditional<F64, double, float>::type;
  Acc acc[TT];
#pragma unroll
  for (int i = 0; i < TT; ++i) acc[i] = Acc(0);
  float wsq = 0.f;
  for (int c0 = lane; c0 < vpr; c0 += 32 * U) {
    if (c0 != lane) {   // the first chunk was prefetched above
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        wv[u] = c < vpr ? wrow[c] : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c >= vpr) break;
      float wf[8];
      unpack8(wv[u], wf);
#pragma unroll
      for (int i = 0; i < 8; ++i) wsq = fmaf(wf[i], wf[i], wsq);
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        float xf[8];
        unpack8(sx[tt * vpr + c], xf);
        if constexpr (ACC == kAccMixed) {
          float p = xf[0] * wf[0];
#pragma unroll
          for (int i = 1; i < 8; ++i) p = fmaf(xf[i], wf[i], p);
          acc[tt] += static_cast<double>(p);
        } else if constexpr (ACC == kAcc64) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[tt] = fma(static_cast<double>(xf[i]), static_cast<double>(wf[i]), acc[tt]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[tt] = fmaf(xf[i], wf[i], acc[tt]);
        }
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    if constexpr (F64)
      acc[tt] = warp_sum_d(acc[tt]);
    else
      acc[tt] = warp_sum(acc[tt]);
  }
  wsq = warp_sum(wsq);
  if (lane == 0) {
    const float b = bias ? bias[e] : 0.f;
    for (int tt = 0; tt < nt; ++tt)
      logits[static_cast<size_t>(t0 + tt) * E + e] = static_cast<float>(acc[tt] + static_cast<Acc>(b));
    if (blockIdx.x == 0 || every_cta_wnorm) wnorm[e] = sqrtf(wsq);
  }
}

template <int TT, int ACC>
__global__ void __launch_bounds__(256) router_logits_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ router_w,
    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits,
    float* __restrict__ xnorm, float* __restrict__ wnorm, float* __restrict__ amax_tok) {
  extern __shared__ uint4 sx[];
  pdl_wait();
  pdl_launch_next();
  logits_body<TT, ACC>(hidden, router_w, bias, T, H, E, logits, xnorm, wnorm, amax_tok, sx);
}

// ---------------------------------------------------------------------------
// Kernel 1b (large batches): the same logits as a register-tiled fp32 SIMT
// GEMM.  CTA = 64 tokens x 64 experts, 256 threads, each thread 4 tokens x 4
// experts; K in tiles of 64 staged as fp32 in smem (converted once per CTA),
// the next tile's bf16 rows prefetched into registers while this one is
// multiplied.  Blocked summation bounds the error: each output sums a tile's
// 64 exact products in one FMA chain (63 roundings) and adds the tile sum to
// its total (H/64 - 1 roundings), so every term sees at most H/64 + 62
// roundings (the bound handed to the top-k kernel uses H/64 + 64).  The
// norms and per-token amax|x| come from the staged values: token rows in the
// CTAs of expert tile 0, router rows in the CTAs of token tile 0.
// Split-K (gridDim.z = S > 1, for batches whose tiles alone would leave SMs
// idle): CTA z covers K tiles [z n/S, (z+1) n/S) and writes its partial
// logits (no bias), partial sums of squares and partial amax to rsplit; the
// top-k kernel adds the S partials in z order, then the bias.  Each term then
// sees at most H/(64S) + S + 61 <= H/64 + 64 roundings.
// ---------------------------------------------------------------------------
constexpr int kLgT = 64;          // tokens per CTA
constexpr int kLgE = 64;          // experts per CTA
constexpr int kLgK = 64;          // K per tile
constexpr int kLgLd = kLgK + 4;   // smem row stride (floats): rows 4 banks apart

__global__ void __launch_bounds__(256) router_logits_tiled_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ router_w,
    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits,
    float* __restrict__ xnorm, float* __restrict__ wnorm, float* __restrict__ amax_tok,
    float* __restrict__ rsplit) {
  extern __shared__ float4 lg_smem[];
  float* xs = reinterpret_cast<float*>(lg_smem);    // [2][kLgT][kLgLd]
  float* wsm = xs + 2 * kLgT * kLgLd;               // [2][kLgE][kLgLd]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kLgT, e0 = blockIdx.y * kLgE;
  const int vpr = H / 8;
  const uint4* hv = reinterpret_cast<const uint4*>(hidden);
  const uint4* rv = reinterpret_cast<const uint4*>(router_w);
  // staging map: 512 16-byte vectors per operand tile, two per thread:
  // row r0 (and r0 + 32), vector q of the row's 8
  const int q = tid & 7, r0 = tid >> 3;
  const bool xrow_ok[2] = {t0 + r0 < T, t0 + r0 + 32 < T};
  const bool wrow_ok[2] = {e0 + r0 < E, e0 + r0 + 32 < E};
  const bool do_xn = blockIdx.y == 0, do_wn = blockIdx.x == 0;
  float xss[2] = {0.f, 0.f}, xam[2] = {0.f, 0.f}, wss[2] = {0.f, 0.f};
  uint4 px[2], pw[2];
  auto fetch = [&](int kt) {
    const int c = kt * (kLgK / 8) + q;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      px[s] = xrow_ok[s] ? hv[static_cast<size_t>(t0 + r0 + 32 * s) * vpr + c] : make_uint4(0, 0, 0, 0);
      pw[s] = wrow_ok[s] ? rv[static_cast<size_t>(e0 + r0 + 32 * s) * vpr + c] : make_uint4(0, 0, 0, 0);
    }
  };
  auto stage = [&](int buf) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      float f[8], g[8];
      unpack8(px[s], f);
      unpack8(pw[s], g);
      if (do_xn) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xss[s] = fmaf(f[i], f[i], xss[s]);
          xam[s] = fmaxf(xam[s], fabsf(f[i]));
        }
      }
      if (do_wn) {
#pragma unroll
        for (int i = 0; i < 8; ++i) wss[s] = fmaf(g[i], g[i], wss[s]);
      }
      float4* dx = reinterpret_cast<float4*>(xs + (buf * kLgT + r0 + 32 * s) * kLgLd + 8 * q);
      float4* dw = reinterpret_cast<float4*>(wsm + (buf * kLgE + r0 + 32 * s) * kLgLd + 8 * q);
      dx[0] = make_float4(f[0], f[1], f[2], f[3]);
      dx[1] = make_float4(f[4], f[5], f[6], f[7]);
      dw[0] = make_float4(g[0], g[1], g[2], g[3]);
      dw[1] = make_float4(g[4], g[5], g[6], g[7]);
    }
  };

  pdl_wait();
  pdl_launch_next();
  // compute map: a warp covers 4 token rows x 8 expert rows, so each of its
  // 16-byte smem loads touches 4 (x) or 8 (w) distinct rows in distinct banks
  const int warp = tid >> 5, lane = tid & 31;
  const int tx = (lane & 7) | ((warp & 1) << 3);   // experts tx + 16 j
  const int ty = (lane >> 3) + 4 * (warp >> 1);    // tokens ty + 16 i
  float acc[4][4], blk[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int S = gridDim.z, z = blockIdx.z;
  const int nkt_all = H / kLgK;
  const int kt0 = z * nkt_all / S, nkt = (z + 1) * nkt_all / S - kt0;
  fetch(kt0);
  stage(0);
  __syncthreads();
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) fetch(kt0 + kt + 1);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) blk[i][j] = 0.f;
    const float* xb = xs + buf * kLgT * kLgLd;
    const float* wb = wsm + buf * kLgE * kLgLd;
#pragma unroll 4
    for (int kq = 0; kq < kLgK / 4; ++kq) {
      float4 xa[4], wa[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) xa[i] = *reinterpret_cast<const float4*>(xb + (ty + 16 * i) * kLgLd + 4 * kq);
#pragma unroll
      for (int j = 0; j < 4; ++j) wa[j] = *reinterpret_cast<const float4*>(wb + (tx + 16 * j) * kLgLd + 4 * kq);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          blk[i][j] = fmaf(xa[i].x, wa[j].x, blk[i][j]);
          blk[i][j] = fmaf(xa[i].y, wa[j].y, blk[i][j]);
          blk[i][j] = fmaf(xa[i].z, wa[j].z, blk[i][j]);
          blk[i][j] = fmaf(xa[i].w, wa[j].w, blk[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += blk[i][j];
    if (kt + 1 < nkt) stage(buf ^ 1);
    __syncthreads();
  }

  // split-K partial regions: logits [S][T][E], sum x^2 [S][T], amax [S][T], sum w^2 [S][E]
  float* p_log = rsplit;
  float* p_xss = rsplit + static_cast<size_t>(S) * T * E;
  float* p_xam = p_xss + static_cast<size_t>(S) * T;
  float* p_wss = p_xam + static_cast<size_t>(S) * T;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + tx + 16 * j;
    if (e >= E) continue;
    const float b = bias ? bias[e] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + ty + 16 * i;
      if (t >= T) continue;
      if (S == 1)
        logits[static_cast<size_t>(t) * E + e] = acc[i][j] + b;
      else
        p_log[(static_cast<size_t>(z) * T + t) * E + e] = acc[i][j];
    }
  }
  // norms: the 8 threads of a staging row are 8 consecutive lanes
#pragma unroll
  for (int s = 0; s < 2; ++s) {
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
      xss[s] += __shfl_xor_sync(0xffffffffu, xss[s], m);
      xam[s] = fmaxf(xam[s], __shfl_xor_sync(0xffffffffu, xam[s], m));
      wss[s] += __shfl_xor_sync(0xffffffffu, wss[s], m);
    }
    if (q == 0) {
      const int t = t0 + r0 + 32 * s, e = e0 + r0 + 32 * s;
      if (do_xn && xrow_ok[s]) {
        if (S == 1) {
          xnorm[t] = sqrtf(xss[s]);
          amax_tok[t] = xam[s];
        } else {
          p_xss[static_cast<size_t>(z) * T + t] = xss[s];
          p_xam[static_cast<size_t>(z) * T + t] = xam[s];
        }
      }
      if (do_wn && wrow_ok[s]) {
        if (S == 1)
          wnorm[e] = sqrtf(wss[s]);
        else
          p_wss[static_cast<size_t>(z) * E + e] = wss[s];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: one warp per token.  fp32 softmax, top-(k+1) by repeated warp
// argmax, certification against the error bound, fallback tiers 2-3.
// kPer = experts per lane (register arrays sized by the expert count).
// gamma: relative summation bound of the logit kernel that ran (times
// sum|x w| <= ||x|| ||w||); ulast: relative error of the last roundings (bias
// add, storage to fp32).
// nsplit > 1: the logits kernel ran split-K; this kernel first adds the
// token's nsplit partial logits in split order, then the bias, stores the
// row to `logits`, and forms ||x_t||, amax|x_t| and ||w_e|| from the partial
// sums.
// ---------------------------------------------------------------------------
// Top-k of token t by the calling warp.  Logits, norms and partials are
// read through L2 (they may come from other CTAs of the same grid).
template <int kPer>
__device__ void topk_token(
    int t, float* __restrict__ logits, float* __restrict__ xnorm, const float* __restrict__ wnorm,
    float* __restrict__ amax_tok, const float* __restrict__ rsplit, int nsplit,
    const float* __restrict__ bias, const __nv_bfloat16* __restrict__ hidden,
    const __nv_bfloat16* __restrict__ router_w, int T, int H, int E, int k, float gamma, float ulast,
    int32_t* __restrict__ topk_ids, float* __restrict__ topk_w, unsigned char* __restrict__ cand,
    uint32_t* __restrict__ hdr, bool tc_tier) {
  const int lane = threadIdx.x & 31;
  const int nper = (E + 31) / 32;
  float* row = logits + static_cast<size_t>(t) * E;
  const float* p_xss = rsplit + static_cast<size_t>(nsplit) * T * E;
  const float* p_xam = p_xss + static_cast<size_t>(nsplit) * T;
  const float* p_wss = p_xam + static_cast<size_t>(nsplit) * T;
  float xn;
  if (nsplit > 1) {
    float ss = 0.f, am = 0.f;
    for (int z = 0; z < nsplit; ++z) {
      ss += __ldcg(p_xss + static_cast<size_t>(z) * T + t);
      am = fmaxf(am, __ldcg(p_xam + static_cast<size_t>(z) * T + t));
    }
    xn = sqrtf(ss);
    if (lane == 0) {
      xnorm[t] = xn;
      amax_tok[t] = am;
    }
    for (int e = lane; e < E; e += 32) {
      float v = __ldcg(rsplit + static_cast<size_t>(t) * E + e);
      for (int z = 1; z < nsplit; ++z) v += __ldcg(rsplit + (static_cast<size_t>(z) * T + t) * E + e);
      row[e] = v + (bias ? bias[e] : 0.f);
    }
    __syncwarp();
  } else {
    xn = __ldcg(xnorm + t);
  }
  auto wnorm_of = [&](int e) -> float {
    if (nsplit <= 1) return __ldcg(wnorm + e);
    float ss = 0.f;
    for (int z = 0; z < nsplit; ++z) ss += __ldcg(p_wss + static_cast<size_t>(z) * E + e);
    return sqrtf(ss);
  };
  // plus H products that might underflow in fp32 (2^-149 each)
  const float tiny = static_cast<float>(H) * 1.4012985e-45f;

  float v[kPer];
  uint32_t taken = 0;
  float rmax = 0.f, vmax = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = -FLT_MAX;
    if (i < nper && e < E) {
      const float lv = __ldcg(row + e);
      v[i] = isnan(lv) ? -FLT_MAX : lv;   // a NaN logit ranks last
      const float b = bias ? fabsf(bias[e]) : 0.f;
      const float r = (gamma * xn * wnorm_of(e) + ulast * (fabsf(v[i]) + b) + tiny) * 1.001f;
      rmax = fmaxf(rmax, r);
      vmax = fmaxf(vmax, v[i]);
    }
  }
  rmax = warp_max(rmax);
  vmax = warp_max(vmax);
  float se = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (i < nper && lane + 32 * i < E) se += expf(v[i] - vmax);
  se = warp_sum(se);

  // top-(k+1) selection, warp-wide argmax per round; slot s is kept by lane
  // s (slot 32, the extra one when k = 32, in a warp-uniform register)
  const int nsel = min(k + 1, E);
  int my_idx = -1;
  float my_v = -FLT_MAX, extra_v = -FLT_MAX;
  for (int s = 0; s < nsel; ++s) {
    float bv = -FLT_MAX;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      if (i < nper && e < E && !((taken >> i) & 1u) && beats(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, m);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, m);
      if (beats(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (s == lane) {
      my_idx = bi;
      my_v = bv;
    }
    if (s == 32) extra_v = bv;
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
  }

  // certified when every adjacent gap among the top k+1 exceeds twice the
  // bound.  tc_tier (logits from the tensor cores, whose bound is loose):
  // every token re-evaluates its candidates, which also yields the weights.
  bool certified = !tc_tier;
  double my_d = 0.0;   // re-evaluated logit of this lane's slot (tc_tier)
  if (certified && rmax > 0.f) {
    const double margin = 2.000001 * static_cast<double>(rmax);
    const float down = __shfl_down_sync(0xffffffffu, my_v, 1);
    const float next_v = lane == 31 ? extra_v : down;
    const bool bad = lane + 1 < nsel &&
                     !(static_cast<double>(my_v) - static_cast<double>(next_v) > margin);
    certified = !__any_sync(0xffffffffu, bad);
  }

  if (!certified) {
    // counted here for CUDA-core logits; from tensor-core logits every token
    // comes here, and only the ones the mixed values leave open are counted
    if (lane == 0 && !tc_tier) atomicAdd(hdr + kHdrUncertain, 1u);
    const float kth_v = __shfl_sync(0xffffffffu, my_v, k - 1);
    int got = 0;
    auto put = [&](int e, double d) {   // slot `got` takes expert e (re-evaluated logit d)
      if (lane == got) {
        my_idx = e;
        const float lv = __ldcg(row + e);
        my_v = isnan(lv) ? -FLT_MAX : lv;
        my_d = d;
      }
      ++got;
    };
    // ---- tier 2: candidates re-evaluated on the CUDA cores ----------------
    int* c_idx = reinterpret_cast<int*>(cand + static_cast<size_t>(t) * E * 16);
    int* c_ord = c_idx + E;
    double* c_val = reinterpret_cast<double*>(c_ord + E);
    const double thr = static_cast<double>(kth_v) - 2.000001 * static_cast<double>(rmax);
    int nc = 0;
    for (int i = 0; i < nper; ++i) {
      const int e = lane + 32 * i;
      const bool is_c = e < E && static_cast<double>(v[i]) >= thr;
      const uint32_t bal = __ballot_sync(0xffffffffu, is_c);
      if (is_c) c_idx[nc + __popc(bal & ((1u << lane) - 1u))] = e;
      nc += __popc(bal);
    }
    __syncwarp();
    const double u32 = 5.9604644775390625e-08, u64 = 1.1102230246251565e-16;
    const __nv_bfloat16* xrow = hidden + static_cast<size_t>(t) * H;
    // every candidate's logit (+ bias) into c_val, ranked; returns the largest bound
    auto evaluate = [&](bool mixed) -> double {
      const double g = mixed ? (7.0 * u32 + (H / 256 + 16) * u64) * 1.0001
                             : static_cast<double>(H / 32 + 16) * u64 * 1.0001;
      const double floor_err = mixed ? static_cast<double>(H) * 3.5032461608120427e-45 : 1e-300;
      double rmx = 0.0;
      for (int c = 0; c < nc; c += 4) {   // four candidates per pass over the row
        const int nw = min(4, nc - c);
        const __nv_bfloat16* wrows[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) wrows[r] = router_w + static_cast<size_t>(c_idx[c + (r < nw ? r : 0)]) * H;
        double dd[4];
        if (mixed)
          logits4<true>(xrow, wrows, nw, H, dd);
        else
          logits4<false>(xrow, wrows, nw, H, dd);
        for (int r = 0; r < nw; ++r) {
          const int e = c_idx[c + r];
          const double b = bias ? static_cast<double>(bias[e]) : 0.0;
          const double d = dd[r] + b;
          rmx = fmax(rmx, (g * xn * wnorm_of(e) + 2.3e-16 * (fabs(d) + fabs(b))) * 1.001 + floor_err);
          if (lane == 0) c_val[c + r] = d;
        }
      }
      __syncwarp();
      rank_candidates(c_idx, c_ord, c_val, nc);
      return rmx;
    };
    // tc_tier: first in mixed precision, which decides when every adjacent
    // gap among the first k+1 exceeds twice its bound; otherwise (and for
    // CUDA-core logits) in fp64
    double margin = 2.000001 * evaluate(tc_tier);
    if (tc_tier) {
      bool bad = false;
      for (int i = lane; i < k && i + 1 < nc; i += 32) bad |= !(c_val[c_ord[i]] - c_val[c_ord[i + 1]] > margin);
      if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0) atomicAdd(hdr + kHdrUncertain, 1u);
        margin = 2.000001 * evaluate(false);
      }
    }
    // ---- tier 3: clusters closer than the margin, ordered exactly ----------
    assemble_in_order(c_idx, c_ord, c_val, nc, k, margin, xrow, router_w, bias, H, got, put);
  }

  // renormalised weights of the selected experts: fp32 softmax values
  // renormalised over the k; on tc_tier the same quantity from the
  // re-evaluated logits, exp(d_j - max_j d) / sum_j (the full softmax's
  // denominator cancels in the renormalisation)
  float p;
  if (tc_tier) {
    double dm = lane < k ? my_d : -1.0e300;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) dm = fmax(dm, __shfl_xor_sync(0xffffffffu, dm, m));
    p = lane < k ? expf(static_cast<float>(my_d - dm)) : 0.f;
  } else {
    p = lane < k ? expf(my_v - vmax) / se : 0.f;
  }
  const float psum = warp_sum(p);
  if (lane < k) {
    topk_ids[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = p / psum;
  }
}

// One warp per token.  With `with_align` (decode-sized calls) the CTA that
// finishes last also runs the align: after a barrier (every top-k of the CTA
// stored) its thread 0 takes an acquire-release ticket of the grid; the CTA
// that draws the last one runs the align in its one-CTA form (its shared
// memory holds the per-warp histograms).  No CTA waits for another; the
// counter is reset by the CTA that completes it, so every call starts at 0.
__device__ __forceinline__ unsigned int ticket_acq_rel(uint32_t* p) {
  unsigned int old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

template <int kPer>
__global__ void __launch_bounds__(256) router_topk_kernel(
    float* __restrict__ logits, float* __restrict__ xnorm, const float* __restrict__ wnorm,
    float* __restrict__ amax_tok, const float* __restrict__ rsplit, int nsplit,
    const float* __restrict__ bias, const __nv_bfloat16* __restrict__ hidden,
    const __nv_bfloat16* __restrict__ router_w, int T, int H, int E, int k, float gamma, float ulast,
    int32_t* __restrict__ topk_ids, float* __restrict__ topk_w, unsigned char* __restrict__ cand,
    uint32_t* __restrict__ hdr, AlignArgs aa, int with_align, int tc_tier) {
  extern __shared__ int align_hist[];
  __shared__ int s_last;
  pdl_wait();
  pdl_launch_next();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t < T)
    topk_token<kPer>(t, logits, xnorm, wnorm, amax_tok, rsplit, nsplit, bias, hidden, router_w, T, H,
                     E, k, gamma, ulast, topk_ids, topk_w, cand, hdr, tc_tier != 0);
  if (!with_align) return;
  __syncthreads();   // every top-k of this CTA is stored
  if (threadIdx.x == 0) {
    uint32_t* cnt = hdr + kHdrRouterAll;
    const bool last = ticket_acq_rel(cnt) == gridDim.x - 1;
    if (last) *cnt = 0u;
    s_last = last ? 1 : 0;
  }
  __syncthreads();
  if (s_last) align_cta(aa, 0, 0, align_hist);
}

// ---------------------------------------------------------------------------
template <int TT, int ACC>
static cudaError_t launch_logits(const RouterArgs& a, cudaStream_t st) {
  auto kern = router_logits_kernel<TT, ACC>;
  const int smem = TT * a.H * 2;
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), smem);
  if (err != cudaSuccess) return err;
  dim3 grid((a.T + TT - 1) / TT, (a.E + 7) / 8);
  return launch_pdl(kern, grid, dim3(256), smem, st, a.hidden, a.router_w, a.bias, a.T, a.H, a.E,
                    a.logits, a.xnorm, a.wnorm, a.amax_tok);
}

template <int kPer>
static cudaError_t launch_topk(const RouterArgs& a, float gamma, float ulast, int nsplit,
                               cudaStream_t st, const AlignArgs* aa = nullptr, bool tc_tier = false) {
  const int smem = aa ? 8 * a.E * 4 : 0;   // the align's per-warp histograms (8 warps)
  auto kern = router_topk_kernel<kPer>;
  if (smem > 0) {
    cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), smem);
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(kern, dim3((a.T + 7) / 8), dim3(256), smem, st, a.logits, a.xnorm, a.wnorm, a.amax_tok,
                    a.rsplit, nsplit, a.bias, a.hidden, a.router_w, a.T, a.H, a.E, a.k, gamma, ulast,
                    a.topk_ids, a.topk_w, a.cand, a.hdr, aa ? *aa : AlignArgs{}, aa ? 1 : 0, tc_tier ? 1 : 0);
}

// ---------------------------------------------------------------------------
// Kernel 1c (batch-invariant calls with small batches): the tiled kernel's
// exact arithmetic (unsplit) at one token per CTA, one expert per warp.  Lane
// l forms the fp32 FMA chains of K tiles l, l + 32, ... (64 products each, in
// K order, from zero); lane 0 then adds the tile sums in K-tile order from
// zero and adds the bias, so every logit is bit-identical to the tiled
// kernel's for any batch size.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_logits_blocked_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ router_w,
    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits,
    float* __restrict__ xnorm, float* __restrict__ wnorm, float* __restrict__ amax_tok) {
  pdl_wait();
  pdl_launch_next();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int e = blockIdx.y * 8 + warp;
  const int vpr = H / 8;
  const int ntiles = H / kLgK;            // 64-element K tiles
  const uint4* xv = reinterpret_cast<const uint4*>(hidden) + static_cast<size_t>(t) * vpr;
  if (blockIdx.y == 0 && warp == 0) {     // ||x_t|| and amax|x_t| (certification, FP8 scale)
    float ss = 0.f, am = 0.f;
    for (int c = lane; c < vpr; c += 32) {
      float f[8];
      unpack8(xv[c], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ss = fmaf(f[i], f[i], ss);
        am = fmaxf(am, fabsf(f[i]));
      }
    }
    ss = warp_sum(ss);
    am = warp_max(am);
    if (lane == 0) {
      xnorm[t] = sqrtf(ss);
      amax_tok[t] = am;
    }
  }
  if (e >= E) return;
  const uint4* wv = reinterpret_cast<const uint4*>(router_w) + static_cast<size_t>(e) * vpr;
  float acc = 0.f, wsq = 0.f;
  for (int j0 = 0; j0 < ntiles; j0 += 32) {
    const int j = j0 + lane;
    float tsum = 0.f;
    if (j < ntiles) {
#pragma unroll
      for (int q = 0; q < kLgK / 8; ++q) {
        float xf[8], wf[8];
        unpack8(xv[j * (kLgK / 8) + q], xf);
        unpack8(wv[j * (kLgK / 8) + q], wf);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          tsum = fmaf(xf[i], wf[i], tsum);
          wsq = fmaf(wf[i], wf[i], wsq);
        }
      }
    }
    // tile sums added in K-tile order by lane 0
    const int nj = min(32, ntiles - j0);
    for (int i = 0; i < nj; ++i) {
      const float v = __shfl_sync(0xffffffffu, tsum, i);
      if (lane == 0) acc += v;
    }
  }
  wsq = warp_sum(wsq);
  if (lane == 0) {
    const float b = bias ? bias[e] : 0.f;
    logits[static_cast<size_t>(t) * E + e] = acc + b;
    if (t == 0) wnorm[e] = sqrtf(wsq);
  }
}

static cudaError_t launch_logits_tiled(const RouterArgs& a, int nsplit, cudaStream_t st) {
  auto kern = router_logits_tiled_kernel;
  const int smem = 2 * (kLgT + kLgE) * kLgLd * 4;
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), smem);
  if (err != cudaSuccess) return err;
  dim3 grid((a.T + kLgT - 1) / kLgT, (a.E + kLgE - 1) / kLgE, nsplit);
  return launch_pdl(kern, grid, dim3(256), smem, st, a.hidden, a.router_w, a.bias, a.T, a.H, a.E,
                    a.logits, a.xnorm, a.wnorm, a.amax_tok, a.rsplit);
}

static bool fuse_align_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MOE_FUSE_ALIGN");
    v = (e && std::atoi(e) == 1) ? 1 : 0;
  }
  return v == 1;
}

cudaError_t launch_router_topk_tc(const RouterArgs& a, float gamma, float ulast, cudaStream_t st,
                                  const AlignArgs* fuse_align, bool* fused) {
  if (fused) *fused = false;
  const AlignArgs* aa = nullptr;
  if (fuse_align_enabled() && fuse_align != nullptr && fused != nullptr && a.E <= 256 &&
      static_cast<long long>(a.T) * a.k < kAlignSliceMin) {
    aa = fuse_align;
    *fused = true;
  }
  // logits from the tensor cores: every token's candidates re-evaluated
  if (a.E <= 64) return launch_topk<2>(a, gamma, ulast, 1, st, aa, true);
  if (a.E <= 128) return launch_topk<4>(a, gamma, ulast, 1, st, aa, true);
  if (a.E <= 256) return launch_topk<8>(a, gamma, ulast, 1, st, aa, true);
  return launch_topk<kMaxExperts / 32>(a, gamma, ulast, 1, st, aa, true);
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t st, const AlignArgs* fuse_align, bool* fused) {
  if (fused) *fused = false;
  // fp64 accumulation while the logit work is small (decode batches); fp32
  // with the wider certified bound for large batches
  // fp64 accumulation while the logit work is small (decode batches): per
  // product up to 2^25 multiply-adds, in 8-product fp32 blocks up to 2^28;
  // fp32 with the wider certified bound for large batches
  const double macs = static_cast<double>(a.T) * a.E * a.H;
  const bool acc64 = macs <= static_cast<double>(1 << 28);
  int mode = !acc64 ? kAcc32 : (macs <= static_cast<double>(1 << 25) ? kAcc64 : kAccMixed);
  cudaError_t err;
  int nchain;
  int nsplit = 1;
  if (a.invariant || (!acc64 && a.E >= 32)) {
    // large batch: register-tiled fp32 GEMM (blocked summation, see above),
    // split over K until the grid fills two CTAs per SM
    const int tiles = ((a.T + kLgT - 1) / kLgT) * ((a.E + kLgE - 1) / kLgE);
    if (a.rsplit != nullptr && !a.invariant) {
      const int want = (2 * current_sm_count() + tiles - 1) / tiles;
      nsplit = want < 1 ? 1 : (want > kRouterSplits ? kRouterSplits : want);
      if (nsplit > a.H / kLgK) nsplit = a.H / kLgK;
    }
    const bool blocked = a.invariant && tiles < current_sm_count();
    if (blocked)   // the same arithmetic, spread over more SMs
      err = launch_pdl(router_logits_blocked_kernel, dim3(a.T, (a.E + 7) / 8), dim3(256), 0, st,
                       a.hidden, a.router_w, a.bias, a.T, a.H, a.E, a.logits, a.xnorm, a.wnorm,
                       a.amax_tok);
    else
      err = launch_logits_tiled(a, nsplit, st);
    nchain = a.H / kLgK + 64;
    mode = kAcc32;
  } else {
    // tokens per CTA: the largest of 16, 8, 4, 2 that still gives two waves
    // of CTAs (fewer tokens per CTA means more re-reads of router rows from
    // L2, but small decode batches need the parallelism), capped by shared
    // memory.  Chain: H/32 FMAs per lane plus the 5-level butterfly.
    const int waves2 = 2 * current_sm_count();
    const int eblocks = (a.E + 7) / 8;
    int tt = 1;
    for (int c = 16; c >= 2; c /= 2) {
      if (c * a.H * 2 <= 200 * 1024 && ((a.T + c - 1) / c) * eblocks >= waves2) {
        tt = c;
        break;
      }
    }
    switch (mode * 32 + tt) {
      case kAcc64 * 32 + 16: err = launch_logits<16, kAcc64>(a, st); break;
      case kAcc64 * 32 + 8: err = launch_logits<8, kAcc64>(a, st); break;
      case kAcc64 * 32 + 4: err = launch_logits<4, kAcc64>(a, st); break;
      case kAcc64 * 32 + 2: err = launch_logits<2, kAcc64>(a, st); break;
      case kAcc64 * 32 + 1: err = launch_logits<1, kAcc64>(a, st); break;
      case kAccMixed * 32 + 16: err = launch_logits<16, kAccMixed>(a, st); break;
      case kAccMixed * 32 + 8: err = launch_logits<8, kAccMixed>(a, st); break;
      case kAccMixed * 32 + 4: err = launch_logits<4, kAccMixed>(a, st); break;
      case kAccMixed * 32 + 2: err = launch_logits<2, kAccMixed>(a, st); break;
      case kAccMixed * 32 + 1: err = launch_logits<1, kAccMixed>(a, st); break;
      case kAcc32 * 32 + 16: err = launch_logits<16, kAcc32>(a, st); break;
      case kAcc32 * 32 + 8: err = launch_logits<8, kAcc32>(a, st); break;
      case kAcc32 * 32 + 4: err = launch_logits<4, kAcc32>(a, st); break;
      case kAcc32 * 32 + 2: err = launch_logits<2, kAcc32>(a, st); break;
      default: err = launch_logits<1, kAcc32>(a, st); break;
    }
    nchain = a.H / 32 + 16;
  }
  if (err != cudaSuccess) return err;
  // relative bounds (unit roundoff u32 = 2^-24, u64 = 2^-53): an fp64 chain
  // of nchain roundings; the mixed form adds a 7-step fp32 chain per 8
  // products; fp32 chains of nchain roundings
  const double u32 = 5.9604644775390625e-08, u64 = 1.1102230246251565e-16;
  const float gamma = mode == kAcc64     ? static_cast<float>(nchain * u64 * 1.0001)
                      : mode == kAccMixed ? static_cast<float>((7.0 * u32 + nchain * u64) * 1.0001)
                                          : static_cast<float>(nchain * u32 * 1.0001);
  const float ulast = mode != kAcc32 ? static_cast<float>(u32) : static_cast<float>(2.0 * u32);
  // MOE_FUSE_ALIGN=1: decode-sized calls let the top-k kernel's last CTA run
  // the align (measurements only: the separate align launch, whose start
  // overlaps the top-k's tail under programmatic launch, measured faster:
  // decode 160.8 -> 155.0 us, tiny 39.1 -> 32.9 us, decode-fp8 unchanged)
  const AlignArgs* aa = nullptr;
  if (fuse_align_enabled() && fuse_align != nullptr && fused != nullptr && a.E <= 256 &&
      static_cast<long long>(a.T) * a.k < kAlignSliceMin) {
    aa = fuse_align;
    *fused = true;
  }
  if (a.E <= 64) return launch_topk<2>(a, gamma, ulast, nsplit, st, aa);
  if (a.E <= 128) return launch_topk<4>(a, gamma, ulast, nsplit, st, aa);
  if (a.E <= 256) return launch_topk<8>(a, gamma, ulast, nsplit, st, aa);
  return launch_topk<kMaxExperts / 32>(a, gamma, ulast, nsplit, st, aa);
}

}  // namespace moe
