// Fused inverse rotary position embedding + per-head FP8 (E4M3) quantisation.
//
// The pages name this kernel as the third fix of the MoE serving work: a fused
// RoPE + FP8 quantisation kernel, per head, whose token count must stay a
// runtime value rather than a compile-time specialisation ("AWS details MoE
// kernel fixes for SageMaker, upstreams them to vLLM", third fix; "AWS Unveils
// MoE Kernel Optimizations...", "Eliminating Triton JIT Recompilation").
// What it computes (the readings of the unstated details):
//   for every token t and head h, with c = cos_tab[pos[t], i], s = sin_tab[pos[t], i]:
//     y[i]       = x[i] * c + x[i + D/2] * s         (i < D/2: the pair of halves,
//     y[i + D/2] = x[i + D/2] * c - x[i] * s          turned by minus the angle)
//   in fp32, each product and each sum rounded separately (no fused
//   multiply-add); scale = fp32(amax|y|) / 448 (amax 0 -> 1); code =
//   E4M3(fp32(y / scale)), round-to-nearest-even, saturating to +-448.
//   A position outside [0, max_pos) yields codes 0 and scale 0.  Inputs are
//   finite (a NaN or an infinity in x gives unspecified codes and scale).
//
// The division without a divide.  The kernel is bound by instruction issue,
// not by HBM, and a correctly rounded fp32 division costs about ten
// instructions per element.  Markstein's theorem (P. Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990; also the Handbook of Floating-Point Arithmetic, division
// with a fused multiply-add) gives the same result in three: with r the
// correctly rounded 1/s and q0 = RN(y r) (within one ulp of y/s), the
// residual e = y - q0 s is exact in one FMA and RN(q0 + e r) is the correctly
// rounded y/s, barring underflow and overflow (checked per head: the divide
// serves scales outside [2^-100, 2^100]).  The kernel runs it on negated
// values, n0 = RN(y * -r), e = RN(n0 s + y), n1 = RN(e * -r + n0) = -RN(y/s),
// which also gives a zero quotient the sign of y (the plain order turns -0
// into +0); the codes of the negated quotients are flipped back with one XOR
// per four codes (E4M3 is sign-magnitude and its rounding symmetric).  The
// two lanes of each step share one packed fp32x2 instruction (sm_100), the
// pair kept in one 64-bit register through the three steps.  The
// rotation stays in scalar multiplies and adds with explicit rounding, so no
// product is fused into the sum.
//
// Layout and work split.  x [T, nH, D] bf16, codes [T, nH, D] E4M3, scales
// [T, nH] fp32, tables [max_pos, D/2] fp32.  A head's D/2 pairs are covered by
// D/16 lanes, each taking 8 consecutive pairs: 16 bytes of each half of x, 32
// bytes of each table row, 8 bytes of codes per half.  A warp takes 512/D
// consecutive heads (the lanes of a head reduce their amax with shuffles), the
// grid strides over the heads, so loads and stores are contiguous 16-byte
// vectors.  The roofline is HBM: per head 2 D bytes of x read, D bytes of
// codes and 4 bytes of scale written (the table rows are shared by a token's
// heads); the kernel runs at about half of it, bound by instruction issue, and
// is held to 40 registers (six CTAs per SM), which outruns the unbounded
// 55-register build despite a few spilled values.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Packed fp32x2 arithmetic on 64-bit registers (lane x in the low half).
__device__ __forceinline__ unsigned long long pack2(float x, float y) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(x), "f"(y));
  return d;
}
__device__ __forceinline__ float2 unpack2(unsigned long long v) {
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(v));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ void bf16x8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

}  // namespace

__global__ void __launch_bounds__(256, 6) inv_rope_fp8_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ pos, const float4* __restrict__ cos_tab,
    const float4* __restrict__ sin_tab, long long n_heads_total, int nH, int D, int max_pos,
    uint2* __restrict__ codes, float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int lph = D / 16;                 // lanes per head (a power of two, 1..32)
  const int hpw = 32 / lph;               // heads per warp
  const int sub = lane / lph, q = lane % lph;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  const int half_v = D / 16;              // 16-byte vectors per half of a head (x, bf16)
  for (long long w = blockIdx.x * static_cast<long long>(blockDim.x / 32) + threadIdx.x / 32;
       w * hpw < n_heads_total; w += warps) {
    const long long hd = w * hpw + sub;   // global head index t * nH + h
    const bool live = hd < n_heads_total;
    const long long t = live ? hd / nH : 0;
    const int p = live ? pos[t] : -1;
    const bool valid = live && p >= 0 && p < max_pos;
    float y0[8], y1[8];
    float amax = 0.f;
    if (valid) {
      const uint4 va = x[hd * (2 * half_v) + q];
      const uint4 vb = x[hd * (2 * half_v) + half_v + q];
      float a[8], b[8];
      bf16x8(va, a);
      bf16x8(vb, b);
      const float4* cr = cos_tab + (static_cast<long long>(p) * D / 2 + 8 * q) / 4;
      const float4* sr = sin_tab + (static_cast<long long>(p) * D / 2 + 8 * q) / 4;
      const float4 c0 = cr[0], c1 = cr[1], s0 = sr[0], s1 = sr[1];
      const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y0[i] = __fadd_rn(__fmul_rn(a[i], c[i]), __fmul_rn(b[i], s[i]));
        y1[i] = __fsub_rn(__fmul_rn(b[i], c[i]), __fmul_rn(a[i], s[i]));
        amax = fmaxf(amax, fmaxf(fabsf(y0[i]), fabsf(y1[i])));
      }
    }
    // amax over the lanes of this head (the lane group is aligned and a power of two)
    for (int m = lph / 2; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    if (!live) continue;
    const float scale = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint2 qa = make_uint2(0u, 0u), qb = make_uint2(0u, 0u);
    if (valid) {
      float d0[8], d1[8];
      if (scale >= 0x1p-100f && scale <= 0x1p100f) {
        const float nr = -__frcp_rn(scale);
        const unsigned long long NR = pack2(nr, nr), SC = pack2(scale, scale);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const unsigned long long Y0 = pack2(y0[i], y0[i + 1]), Y1 = pack2(y1[i], y1[i + 1]);
          const unsigned long long n0 = mul2(Y0, NR), n1 = mul2(Y1, NR);
          const unsigned long long e0 = fma2(n0, SC, Y0), e1 = fma2(n1, SC, Y1);
          const float2 q0 = unpack2(fma2(e0, NR, n0)), q1 = unpack2(fma2(e1, NR, n1));
          d0[i] = q0.x; d0[i + 1] = q0.y; d1[i] = q1.x; d1[i + 1] = q1.y;
        }
        qa = make_uint2(e4m3x4(d0[0], d0[1], d0[2], d0[3]) ^ 0x80808080u,
                        e4m3x4(d0[4], d0[5], d0[6], d0[7]) ^ 0x80808080u);
        qb = make_uint2(e4m3x4(d1[0], d1[1], d1[2], d1[3]) ^ 0x80808080u,
                        e4m3x4(d1[4], d1[5], d1[6], d1[7]) ^ 0x80808080u);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          d0[i] = __fdiv_rn(y0[i], scale);
          d1[i] = __fdiv_rn(y1[i], scale);
        }
        qa = make_uint2(e4m3x4(d0[0], d0[1], d0[2], d0[3]), e4m3x4(d0[4], d0[5], d0[6], d0[7]));
        qb = make_uint2(e4m3x4(d1[0], d1[1], d1[2], d1[3]), e4m3x4(d1[4], d1[5], d1[6], d1[7]));
      }
    }
    codes[hd * (2 * half_v) + q] = qa;
    codes[hd * (2 * half_v) + half_v + q] = qb;
    if (q == 0) scales[hd] = valid ? scale : 0.f;
  }
}

cudaError_t launch_inv_rope_fp8(const void* x, const int32_t* pos, const float* cos_tab, const float* sin_tab,
                                int T, int nH, int D, int max_pos, uint8_t* codes, float* scales,
                                cudaStream_t st) {
  const long long heads = static_cast<long long>(T) * nH;
  const int hpw = 512 / D;
  const long long warps = (heads + hpw - 1) / hpw;
  const long long blocks = (warps + 7) / 8;
  const int grid = static_cast<int>(blocks < current_sm_count() * 16LL ? blocks : current_sm_count() * 16LL);
  inv_rope_fp8_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(
      static_cast<const uint4*>(x), pos, reinterpret_cast<const float4*>(cos_tab),
      reinterpret_cast<const float4*>(sin_tab), heads, nH, D, max_pos, reinterpret_cast<uint2*>(codes),
      scales);
  return cudaGetLastError();
}

}  // namespace moe
