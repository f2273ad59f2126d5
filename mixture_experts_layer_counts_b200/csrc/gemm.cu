// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// operands streamed into shared memory by TMA, persistent CTAs (one per SM).
//
// Orientation.  The Hopper "Swap-AB" fix described for vLLM's fused MoE
// ("AWS details MoE kernel fixes for SageMaker...", body; "AWS Unveils MoE
// Kernel Optimizations...", Swap-AB section) computes B^T A^T so the large
// expert-weight dimension fills the instruction's fixed 64-row slot when a
// decode batch has only a handful of tokens.  The sm_100a analogue:
//   kSwap   : A (M = 128) = expert weight rows, B (N = 16..64) = the expert's
//             tokens, D[weight row, token] in TMEM.  Used for experts with few
//             tokens: every weight byte is streamed once, the MMA N is the
//             token count rounded up to 16.
//   kNormal : A (M = 128) = 128 tokens of one expert, B (N = 256) = weight
//             rows, D[token, weight row].  Used for experts with many tokens
//             (prefill-sized batches), where the MMA tile is full.  The
//             gate/up GEMM stages two 128-token M tiles (a 256-token chunk)
//             per weight tile, so each staged weight byte feeds two MMAs.
// Projections.
//   kW13 : gate rows [i, i+.) and up rows [I+i, I+i+.) of w13[e] in two
//          accumulators (swap-AB: two MMAs; normal: one N = 256 MMA over the
//          adjacent gate and up tiles), so one thread holds g and u of the
//          same (token, i) and the epilogue forms h = SiLU(g) * u directly:
//          bf16 path -> inter (bf16, RNE); FP8 path -> h (fp32) + per-CTA
//          amax|h|, and the last gate/up launch of the call closes with a
//          grid barrier and the per-tensor E4M3 requantisation of h
//          (requant_tail), so no separate pass is launched.
//   kW2  : one accumulator; the epilogue multiplies by the router weight
//          w[t, j] and writes the fp32 row to ysc[t*k + j] (its slot), which
//          the combine pass sums in slot order: deterministic, no atomics.
//
// Work split.  A "unit" is one output tile (token chunk x weight-row tile)
// and needs `katoms` K atoms.
//   Swap-AB (HBM-bound): the nunits * katoms atoms are cut into G equal
//   contiguous ranges, one per CTA, so every SM streams the same number of
//   weight bytes whatever the number of active experts.  A unit cut by a
//   range boundary is finished by the CTA that holds its first atoms (the
//   "head", whose range ends there, so it reaches that unit last): the CTAs
//   holding the later atoms write their fp32 partial accumulators to their
//   own slot and raise a flag; the head adds the partials in K order and runs
//   the epilogue.  Fixed order, no atomics on data.
//   Normal (tensor-bound), and swap-AB in the batch-invariant mode: whole
//   units dealt round-robin; normal units ordered expert -> weight tile ->
//   token chunk, so the chunks sharing a weight tile run on neighbouring SMs
//   at the same time and the tile is read from DRAM about once.
//
// Pipeline per CTA:
//   warp 0 lane 0  TMA producer: STAGES-deep ring of {A, B} tiles, 128-byte
//                  K atoms in the 128B-swizzle layout, mbarrier complete_tx.
//                  The tile schedule is complete when the kernel starts, so
//                  the first stages' weight tiles are requested before the
//                  wait for the previous kernel's activations.
//   warp 1 lane 0  MMA issuer: 4 MMAs (K = 16 bf16 / 32 E4M3 each) per atom
//                  and accumulator; tcgen05.commit frees the smem slot; a
//                  final commit hands the TMEM buffer to the epilogue.
//   warps 2..      epilogue (4 warps for swap-AB, 8 for normal: two per TMEM
//                  lane quadrant, warp w reads lanes 32*(w%4)..+31):
//                  tcgen05.ld, math, stores (normal: staged through smem so
//                  whole row segments are written).
// TMEM: two accumulator buffers (the epilogue of one unit overlaps the
// mainloop of the next), except the 256-token gate/up units, whose two M
// tiles fill all 512 columns.  Every wait is bounded (see mbar_wait).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdlib>

#include "common.cuh"
#include "gemm_dev.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

// KA = K atoms per pipeline stage (each weight row then contributes KA*128
// contiguous bytes per stage); BNT = largest token chunk of the swap-AB form.
template <Orient O, Proj P, bool FP8, int KA, int BNT>
struct Cfg {
  static constexpr bool kSwap = O == Orient::kSwap;
  static constexpr bool kDual = P == Proj::kW13;
  // normal-orientation gate/up GEMM: a unit is a 256-token chunk (two M
  // tiles) x one weight tile, so each weight byte staged feeds two MMAs
  // gate/up always; down GEMM when launched with BNT == kPairTokens
  static constexpr bool kPair = !kSwap && (kDual || BNT == kPairTokens);
  static constexpr int kChunkTokens = kPair ? kPairTokens : kNormalTokens;
  static constexpr int kBN = kSwap ? BNT : (kDual ? 128 : 256);   // max N
  static constexpr int kATile = kTileM * kAtomBytes;
  static constexpr int kBTile = kBN * kAtomBytes;
  // swap-AB w13: A = gate and up weight tiles; pair: A = the two token tiles
  static constexpr int kNumA = ((kSwap && kDual) || kPair) ? 2 : 1;
  static constexpr int kNumB = (!kSwap && kDual) ? 2 : 1;
  static constexpr int kBOff = kNumA * kATile;                        // B within an atom set
  static constexpr int kAtomSet = kNumA * kATile + kNumB * kBTile;   // one K atom of every operand
  static constexpr int kStageBytes = KA * kAtomSet;
  // epilogue warps: 4 (one per TMEM lane quadrant); the normal orientation
  // uses 8, two per quadrant, each taking half of the tile's columns
  static constexpr int kEpiWarps = kSwap ? 4 : 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  // normal orientation: per epilogue warp a 32-row x 16-column block (rows
  // padded to 20 words) for the coalesced store transposition
  static constexpr int kEpiCols = 16;
  static constexpr int kEpiLd = 20;
  static constexpr int kEpiBytes = kSwap ? 0 : kEpiWarps * 32 * kEpiLd * 4;
  static constexpr int kStagesFit = (232448 - 1280 - kEpiBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kNumAcc = kDual ? 2 : 1;
  static constexpr int kAccCols = kNumAcc * kBN * (kPair ? 2 : 1);   // per TMEM buffer
  static constexpr int kAccBufs = kPair ? 1 : 2;               // pair: 512 columns, one buffer
  static constexpr int kTmemCols = kAccBufs * kAccCols;        // 128, 256 or 512
  static constexpr int kSmemBytes =
      kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/ + kEpiBytes;
  static constexpr int kAtomElems = FP8 ? 128 : 64;
  static constexpr int kSlotFloats = kNumAcc * kTileM * kBN;   // one CTA's partial tile
  static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                "TMEM allocations are powers of two from 32 to 512 columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kSlotFloats <= kPartialSlotFloats, "partial slot");
  static_assert(kStages >= 2, "pipeline depth");
};

template <Orient O, Proj P, bool FP8, int KA, int BNT>
__global__ void __launch_bounds__((Cfg<O, P, FP8, KA, BNT>::kThreads), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x, const GemmArgs a) {
  using C = Cfg<O, P, FP8, KA, BNT>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 2);   // per epilogue warp amax (<= 8)
  float* epi = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // prologue (overlaps the previous kernel's tail under programmatic launch)
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * C::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    for (int w = 0; w < C::kEpiWarps; ++w) red[w] = 0.f;
    fence_barrier_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The tile schedule comes from the align kernel, which has completed by
  // the time this grid is launched: the kernel before this one (gather,
  // requant or an earlier GEMM) starts its dependents only after its own
  // wait for its predecessors.  So the schedule may be read, and the weight
  // tiles (inputs of the call, written by no kernel) fetched, before the wait
  // for the previous kernel's activations.
  const long long nchunks =
      a.dense_T > 0 ? (a.dense_T + a.dense_chunk - 1) / a.dense_chunk
                    : static_cast<long long>(*reinterpret_cast<const volatile uint32_t*>(a.nchunks));
  const long long nunits = nchunks * a.mtiles;
  const int ksteps = a.katoms / KA;   // pipeline stages per unit
  const long long W = nunits * ksteps;
  // Swap-AB: contiguous balanced atom ranges (units may be split across CTAs).
  // Normal orientation: whole units dealt round-robin in the grouped order.
  constexpr bool kRR = !C::kSwap;   // grouped unit order (normal orientation)
  const bool rr = kRR || a.whole_units != 0;
  // swap-AB token columns of a chunk of nv tokens: rounded up to 16, or the
  // largest chunk when every element must see the same MMA shape
  auto swap_cols = [&](int nv) {
    return a.whole_units ? C::kBN : (nv + kTokenBox - 1) / kTokenBox * kTokenBox;
  };
  int G = static_cast<int>(W / kMinAtomsPerCta);
  G = G < 1 ? 1 : (G > static_cast<int>(gridDim.x) ? static_cast<int>(gridDim.x) : G);
  const bool active = rr ? static_cast<long long>(blockIdx.x) < nunits
                          : (W > 0 && static_cast<int>(blockIdx.x) < G);
  const long long my_a0 = (active && !rr) ? range_begin(W, G, blockIdx.x) : 0;
  const long long my_a1 = (active && !rr) ? range_begin(W, G, blockIdx.x + 1) : 0;
  const Segments seg0{my_a0, my_a1, ksteps, rr, static_cast<long long>(blockIdx.x), nunits,
                      static_cast<int>(gridDim.x)};

  const bool producer = warp == 0 && lane == 0 && active;
  if (!producer) {   // every other thread waits for the previous kernel at once
    grid_dependency_wait();
    grid_dependents_launch();
  }

  if (producer) {
    // ------------------------------------------------------- TMA producer --
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    uint32_t armed = 0, armed_parity = 0;   // per-stage bookkeeping for the abort drain
    // Copies of one pipeline stage: kb = K step of unit u; bit 0 of `parts`
    // issues the weight tiles, bit 1 the token tiles.  Failure-path test:
    // CTA 0 issues nothing for its first stage, so a bounded wait runs out.
    auto issue = [&](int stage, int u, int kb, bool first, int parts) {
      int4 ch;
      int mt;
      unit_coords<kRR, C::kChunkTokens>(a, u, ch, mt);
      const int e = ch.x, p0 = ch.y, nv = ch.z;
      const int wrow0 = e * a.w_rows_per_expert + mt * (C::kSwap ? kTileM : C::kBN);
      const int nbox = C::kSwap ? swap_cols(nv) / kTokenBox : 0;
      if (a.inject_stall != 0 && blockIdx.x == 0 && first) return;
      uint8_t* st = tiles + stage * C::kStageBytes;
#pragma unroll
      for (int ka = 0; ka < KA; ++ka) {
        uint8_t* sa = st + ka * C::kAtomSet;
        const int kc = (kb * KA + ka) * C::kAtomElems;
        if constexpr (C::kSwap) {
          if (parts & 1) {
            tma_load_2d(sa, &tm_w, &full[stage], kc, wrow0, pol_w);
            if constexpr (C::kDual) tma_load_2d(sa + C::kATile, &tm_w, &full[stage], kc, wrow0 + a.up_offset, pol_w);
          }
          if (parts & 2) {
            uint8_t* sb = sa + C::kNumA * C::kATile;
            for (int q = 0; q < nbox; ++q)
              tma_load_2d(sb + q * kTokenBox * kAtomBytes, &tm_x, &full[stage], kc, p0 + q * kTokenBox, pol_x);
          }
        } else {
          if (parts & 2) {
            tma_load_2d(sa, &tm_x, &full[stage], kc, p0, pol_x);
            if constexpr (C::kPair)   // second M tile only when the chunk has one
              if (nv > kTileM) tma_load_2d(sa + C::kATile, &tm_x, &full[stage], kc, p0 + kTileM, pol_x);
          }
          if (parts & 1) {
            tma_load_2d(sa + C::kBOff, &tm_w, &full[stage], kc, wrow0, pol_w);
            if constexpr (C::kDual)
              tma_load_2d(sa + C::kBOff + C::kBTile, &tm_w, &full[stage], kc, wrow0 + a.up_offset, pol_w);
          }
        }
      }
    };
    auto stage_bytes = [&](int u) -> uint32_t {
      if constexpr (C::kSwap) {
        int4 ch;
        int mt;
        unit_coords<kRR, C::kChunkTokens>(a, u, ch, mt);
        const int nvpad = swap_cols(ch.z);
        return KA * (C::kNumA * C::kATile + nvpad * kAtomBytes);
      } else if constexpr (C::kPair) {
        int4 ch;
        int mt;
        unit_coords<kRR, C::kChunkTokens>(a, u, ch, mt);
        return ch.z > kTileM ? C::kStageBytes : C::kStageBytes - KA * C::kATile;
      } else {
        return C::kStageBytes;
      }
    };

    // (1) before the wait: arm the first kStages stages, fetch their weights
    int pre = 0;
    {
      Segments seg = seg0;
      int u, kb0, kb1;
      while (pre < C::kStages && seg.next(u, kb0, kb1)) {
        const uint32_t bytes = stage_bytes(u);
        for (int kb = kb0; kb < kb1 && pre < C::kStages; ++kb, ++pre) {
          mbar_arrive_expect_tx(&full[pre], bytes);
          armed |= 1u << pre;
          issue(pre, u, kb, pre == 0, 1);
        }
      }
    }
    grid_dependency_wait();
    grid_dependents_launch();

    // (2) the token tiles of those stages, then the steady-state pipeline
    int stage = 0;
    uint32_t phase = 0;
    int n = 0;
    bool ok = true;
    Segments seg = seg0;
    int u, kb0, kb1;
    while (ok && seg.next(u, kb0, kb1)) {
      const uint32_t bytes = stage_bytes(u);
      for (int kb = kb0; kb < kb1; ++kb, ++n) {
        if (n < pre) {
          issue(stage, u, kb, n == 0, 2);
        } else {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.hdr, kSiteProducerEmpty, a.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          issue(stage, u, kb, false, 3);
        }
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      // let copies already in flight land before the CTA's smem is released
      int dummy = 0;
      for (int s = 0; s < C::kStages; ++s)
        if ((armed >> s) & 1u)
          mbar_wait(&full[s], (armed_parity >> s) & 1u, reinterpret_cast<volatile int*>(&dummy),
                    a.hdr, kSiteDrainTma, a.timeout_ns);
    }
  } else if (warp == 1 && lane == 0 && active) {
    // ---------------------------------------------------------- MMA issuer --
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    bool issued = false;
    Segments seg = seg0;
    int u, kb0, kb1;
    while (ok && seg.next(u, kb0, kb1)) {
      const int buf = it % C::kAccBufs;
      const uint32_t accph = (it / C::kAccBufs) & 1;
      ++it;
      if (!mbar_wait(&acc_empty[buf], accph ^ 1u, abort_flag, a.hdr, kSiteMmaAccEmpty, a.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int4 ch;
      int mt;
      unit_coords<kRR, C::kChunkTokens>(a, u, ch, mt);
      int n;
      if constexpr (C::kSwap) {
        n = swap_cols(ch.z);
      } else {
        n = C::kNumAcc * C::kBN;   // 256: w13 gate + up in one MMA, w2 one tile
      }
      const uint32_t idesc = idesc_f32acc(FP8 ? 0u : 1u, kTileM, static_cast<uint32_t>(n));
      const uint32_t d0 = tmem_base + buf * C::kAccCols;
      const uint32_t d1 = d0 + C::kBN;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, a.hdr, kSiteMmaFull, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kq = 0; kq < KA * (kAtomBytes / 32); ++kq) {
          const int ka = kq / (kAtomBytes / 32), kk = kq % (kAtomBytes / 32);
          const uint32_t st = smem_u32(tiles + stage * C::kStageBytes + ka * C::kAtomSet);
          const uint32_t acc = (kb > kb0 || kq > 0) ? 1u : 0u;
          const uint32_t off = kk * 32;
          if constexpr (C::kSwap) {
            const uint32_t sb = st + C::kNumA * C::kATile;
            mma_ss<FP8>(d0, sdesc_sw128(st + off), sdesc_sw128(sb + off), idesc, acc);
            if constexpr (C::kDual)
              mma_ss<FP8>(d1, sdesc_sw128(st + C::kATile + off), sdesc_sw128(sb + off), idesc, acc);
          } else {
            // w13: the gate and up tiles are adjacent in smem, so one MMA with
            // N = 2 * kBN covers both; its columns [0, kBN) are the gate
            // accumulator and [kBN, 2 kBN) the up accumulator.  Pair: the
            // second token tile accumulates into the next 2 * kBN columns.
            mma_ss<FP8>(d0, sdesc_sw128(st + off), sdesc_sw128(st + C::kBOff + off), idesc, acc);
            if constexpr (C::kPair)
              if (ch.z > kTileM)
                mma_ss<FP8>(d0 + C::kNumAcc * C::kBN, sdesc_sw128(st + C::kATile + off),
                            sdesc_sw128(st + C::kBOff + off), idesc, acc);
          }
        }
        issued = true;
        mma_commit(&empty[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) mma_commit(&acc_full[buf]);
    }
    if (!ok && issued) {
      int dummy = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), a.hdr, kSiteDrainMma, a.timeout_ns);
    }
  } else if (warp >= 2 && active) {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;               // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;        // accumulator row held by this thread
    float amax = 0.f;
    int it = 0;
    if (a.dense_T > 0 && a.xnorm != nullptr) {
      // router logits: while the first tiles stream in, these warps write the
      // norms (and amax) of a share of the router rows and, when norm_x is
      // given, of the token rows, strided over the active CTAs (0 .. nact-1;
      // the others run no epilogue)
      const int vpr = a.norm_H / 8;
      const long long rows = static_cast<long long>(a.dense_T) + a.n_cols;
      const long long first = a.norm_x != nullptr ? 0 : a.dense_T;
      const long long nact = rr ? (nunits < gridDim.x ? nunits : static_cast<long long>(gridDim.x)) : G;
      for (long long r = first + static_cast<long long>(blockIdx.x) * C::kEpiWarps + (warp - 2); r < rows;
           r += nact * C::kEpiWarps) {
        const bool tok = r < a.dense_T;
        const uint4* src = static_cast<const uint4*>(tok ? a.norm_x : a.norm_w) +
                           static_cast<size_t>(tok ? r : r - a.dense_T) * vpr;
        float ss = 0.f, am = 0.f;
        for (int c0 = lane; c0 < vpr; c0 += 32 * 8) {   // eight 16-byte loads in flight per lane
          uint4 v4[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = c0 + 32 * u;
            v4[u] = c < vpr ? src[c] : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v4[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f2 = __bfloat1622float2(b2[i]);
              ss = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, ss));
              am = fmaxf(am, fmaxf(fabsf(f2.x), fabsf(f2.y)));
            }
          }
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
          ss += __shfl_xor_sync(0xffffffffu, ss, m);
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
        }
        if (lane == 0) {
          if (tok) {
            a.xnorm[r] = sqrtf(ss);
            a.amax_tok[r] = am;
          } else {
            a.wnorm[r - a.dense_T] = sqrtf(ss);
          }
        }
      }
    }
    Segments seg = seg0;
    int u, kb0, kb1;
    while (seg.next(u, kb0, kb1)) {
      const int buf = it % C::kAccBufs;
      const uint32_t accph = (it / C::kAccBufs) & 1;
      ++it;
      if (!mbar_wait(&acc_full[buf], accph, abort_flag, a.hdr, kSiteEpiAccFull, a.timeout_ns)) break;
      tc_fence_after();
      int4 ch;
      int mt;
      unit_coords<kRR, C::kChunkTokens>(a, u, ch, mt);
      const int e = ch.x, p0 = ch.y, nv = ch.z;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      const int ncols = C::kSwap ? swap_cols(nv) : C::kBN;

      if (!rr && kb0 > 0) {   // (whole units only in the round-robin schedule)
        // ---- later piece of a split unit: hand the raw accumulator over ----
        float* slot = a.partials + static_cast<size_t>(blockIdx.x) * kPartialSlotFloats;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[C::kNumAcc][16];
          if constexpr (C::kDual)
            tmem_ld16x2_wait(tbase + c0, tbase + C::kBN + c0, v[0], v[1]);
          else
            tmem_ld16_wait(tbase + c0, v[0]);
#pragma unroll
          for (int ac = 0; ac < C::kNumAcc; ++ac) {
            float4* dst = reinterpret_cast<float4*>(slot + (static_cast<size_t>(ac) * kTileM + row) * C::kBN + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              __stcg(dst + j, make_float4(v[ac][4 * j], v[ac][4 * j + 1], v[ac][4 * j + 2], v[ac][4 * j + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
        __threadfence();
        epilogue_bar<32 * C::kEpiWarps>();
        if (row == 0) st_release(a.flags + blockIdx.x, 1);
        continue;
      }

      // ---- first atoms of the unit: collect the later pieces, then finish ----
      int last = blockIdx.x;
      if (!rr && kb1 < ksteps) {
        const long long unit_end = (static_cast<long long>(u) + 1) * ksteps;
        last = atom_owner(unit_end - 1, W, G);
        bool ok = true;
        for (int c2 = blockIdx.x + 1; c2 <= last && ok; ++c2) ok = wait_flag(a.flags + c2, abort_flag, a.hdr, a.timeout_ns);
        if (!ok) break;
      }
      auto add_partials = [&](float (&v)[C::kNumAcc][16], int c0) {
        for (int c2 = blockIdx.x + 1; c2 <= last; ++c2) {
          const float* slot = a.partials + static_cast<size_t>(c2) * kPartialSlotFloats;
#pragma unroll
          for (int ac = 0; ac < C::kNumAcc; ++ac) {
            const float4* src = reinterpret_cast<const float4*>(slot + (static_cast<size_t>(ac) * kTileM + row) * C::kBN + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 p = __ldcg(src + j);
              v[ac][4 * j] += p.x;
              v[ac][4 * j + 1] += p.y;
              v[ac][4 * j + 2] += p.z;
              v[ac][4 * j + 3] += p.w;
            }
          }
        }
      };

      float scale = 1.f;
      if constexpr (FP8) scale = a.wscale[e] * __uint_as_float(*a.act_scale);

      if constexpr (C::kSwap && C::kDual) {
        const int irow = mt * kTileM + row;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[2][16];
          tmem_ld16x2_wait(tbase + c0, tbase + C::kBN + c0, v[0], v[1]);
          add_partials(v, c0);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < nv) {
              const float gg = v[0][j] * scale, uv = v[1][j] * scale;
              const float h = __fdividef(gg, 1.0f + __expf(-gg)) * uv;
              const size_t o = static_cast<size_t>(p0 + n) * a.ld_out + irow;
              if constexpr (FP8) {
                static_cast<float*>(a.out)[o] = h;
                amax = fmaxf(amax, fabsf(h));
              } else {
                static_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16_rn(h);
              }
            }
          }
        }
      } else if constexpr (C::kSwap) {
        const int hrow = mt * kTileM + row;
        if (a.dense_T > 0) {
          // router logits: row = expert, column n = token p0 + n
          const bool live = hrow < a.n_cols;
          const float b = (live && a.col_bias != nullptr) ? a.col_bias[hrow] : 0.f;
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float v[1][16];
            tmem_ld16_wait(tbase + c0, v[0]);
            add_partials(v, c0);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = c0 + j;
              if (live && n < nv)
                static_cast<float*>(a.out)[static_cast<size_t>(p0 + n) * a.ld_out + hrow] = v[0][j] + b;
            }
          }
        } else {
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float v[1][16];
            tmem_ld16_wait(tbase + c0, v[0]);
            add_partials(v, c0);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = c0 + j;
              const int f = n < nv ? a.perm[p0 + n] : -1;
              if (f >= 0 && f < a.num_assign) {
                const float wt = a.topk_w[f];
                static_cast<float*>(a.out)[static_cast<size_t>(f) * a.ld_out + hrow] = v[0][j] * scale * wt;
              }
            }
          }
        }
      } else if constexpr (C::kDual) {
        // normal w13 (pair): warp half hx takes token rows hx*128 + q*32 +
        // lane of the 256-token chunk, whose gate and up accumulators sit at
        // columns hx*2*kBN + [0, kBN) and + [kBN, 2 kBN).  Each 16-column
        // piece of the warp's 32 rows is staged in smem, then written as
        // whole row segments (bf16: 32 B, fp32: 64 B) with coalesced stores.
        float* sw = epi + (warp - 2) * 32 * C::kEpiLd;
        const int i0 = mt * C::kBN;
        const int hx = (warp - 2) >> 2;
        const int rb = hx * kTileM + q * 32;   // first chunk row of this warp's block
        const bool my_valid = rb + lane < nv;
        const uint32_t th = tbase + hx * 2 * C::kBN;
        for (int c0 = 0; c0 < (rb < nv ? C::kBN : 0); c0 += C::kEpiCols) {
          float v[2][16];
          tmem_ld16x2_wait(th + c0, th + C::kBN + c0, v[0], v[1]);
          float h[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float gg = v[0][j] * scale, uv = v[1][j] * scale;
            h[j] = __fdividef(gg, 1.0f + __expf(-gg)) * uv;
          }
          if constexpr (FP8) {
            if (my_valid) {
#pragma unroll
              for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(h[j]));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<float4*>(sw + lane * C::kEpiLd + 4 * j) =
                  make_float4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
            __syncwarp();
            // 4 lanes per row (64 B), 8 rows per instruction
#pragma unroll
            for (int r0 = 0; r0 < 32; r0 += 8) {
              const int r = r0 + (lane >> 2);
              const float4 val = *reinterpret_cast<const float4*>(sw + r * C::kEpiLd + 4 * (lane & 3));
              if (rb + r < nv)
                *reinterpret_cast<float4*>(static_cast<float*>(a.out) +
                                           static_cast<size_t>(p0 + rb + r) * a.ld_out + i0 + c0 +
                                           4 * (lane & 3)) = val;
            }
          } else {
            uint32_t* su = reinterpret_cast<uint32_t*>(sw);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              uint32_t w4[4];
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(h[8 * j + 2 * m], h[8 * j + 2 * m + 1]);
                w4[m] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(su + lane * C::kEpiLd + 4 * j) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            __syncwarp();
            // 2 lanes per row (32 B), 16 rows per instruction
#pragma unroll
            for (int r0 = 0; r0 < 32; r0 += 16) {
              const int r = r0 + (lane >> 1);
              const uint4 val = *reinterpret_cast<const uint4*>(su + r * C::kEpiLd + 4 * (lane & 1));
              if (rb + r < nv)
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                          static_cast<size_t>(p0 + rb + r) * a.ld_out + i0 + c0 +
                                          8 * (lane & 1)) = val;
            }
          }
          __syncwarp();
        }
      } else if constexpr (C::kPair) {
        // normal w2, 256-token chunk: warp half hx takes token rows
        // hx*128 + q*32 + lane (M tile hx, whose accumulator sits at columns
        // hx*kBN + [0, kBN)), all kBN columns, staged per warp like the w13
        // epilogue; router-weighted fp32 rows to their slot rows f of ysc.
        float* sw = epi + (warp - 2) * 32 * C::kEpiLd;
        const int hx = (warp - 2) >> 2;
        const int rb = hx * kTileM + q * 32;
        const int f = rb + lane < nv ? a.perm[p0 + rb + lane] : -1;
        const bool valid = f >= 0 && f < a.num_assign;
        const float wt = valid ? a.topk_w[f] * scale : 0.f;
        const int h0 = mt * C::kBN;
        const uint32_t th = tbase + hx * C::kBN;
        for (int c0 = 0; c0 < (rb < nv ? C::kBN : 0); c0 += C::kEpiCols) {
          float v[16];
          tmem_ld16_wait(th + c0, v);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4*>(sw + lane * C::kEpiLd + 4 * j) =
                make_float4(v[4 * j] * wt, v[4 * j + 1] * wt, v[4 * j + 2] * wt, v[4 * j + 3] * wt);
          __syncwarp();
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 8) {
            const int r = r0 + (lane >> 2);
            const int fr = __shfl_sync(0xffffffffu, f, r);
            const float4 val = *reinterpret_cast<const float4*>(sw + r * C::kEpiLd + 4 * (lane & 3));
            if (fr >= 0 && fr < a.num_assign)
              __stcs(reinterpret_cast<float4*>(static_cast<float*>(a.out) + static_cast<size_t>(fr) * a.ld_out +
                                               h0 + c0 + 4 * (lane & 3)), val);
          }
          __syncwarp();
        }
      } else {
        // normal w2: router-weighted fp32 rows of the unit's tokens, each to
        // its slot row f of ysc; warp half hx takes columns
        // [hx kBN/2, (hx+1) kBN/2), staged per warp like the w13 epilogue.
        float* sw = epi + (warp - 2) * 32 * C::kEpiLd;
        const int f = row < nv ? a.perm[p0 + row] : -1;
        const bool valid = f >= 0 && f < a.num_assign;
        const float wt = valid ? a.topk_w[f] * scale : 0.f;
        const int h0 = mt * C::kBN;
        const int hx = (warp - 2) >> 2;
        for (int c0 = hx * (C::kBN / 2); c0 < (hx + 1) * (C::kBN / 2); c0 += C::kEpiCols) {
          float v[16];
          tmem_ld16_wait(tbase + c0, v);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4*>(sw + lane * C::kEpiLd + 4 * j) =
                make_float4(v[4 * j] * wt, v[4 * j + 1] * wt, v[4 * j + 2] * wt, v[4 * j + 3] * wt);
          __syncwarp();
          // 4 lanes per row (64 B), 8 rows per instruction
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 8) {
            const int r = r0 + (lane >> 2);
            const int fr = __shfl_sync(0xffffffffu, f, r);
            const float4 val = *reinterpret_cast<const float4*>(sw + r * C::kEpiLd + 4 * (lane & 3));
            // streaming store (evict-first): the T*k fp32 rows are read once, by
            // the combine pass, and should not push weight and token tiles
            // that other CTAs still need out of L2
            if (fr >= 0 && fr < a.num_assign)
              __stcs(reinterpret_cast<float4*>(static_cast<float*>(a.out) + static_cast<size_t>(fr) * a.ld_out +
                                               h0 + c0 + 4 * (lane & 3)), val);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if constexpr (FP8 && C::kDual) {
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
      if (lane == 0) red[warp - 2] = amax;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (FP8 && C::kDual) {
    // every CTA of the grid writes its slot (0 when it had no work)
    if (threadIdx.x == 0) {
      float m = 0.f;
      for (int w = 0; w < C::kEpiWarps; ++w) m = fmaxf(m, red[w]);
      a.amax_cta[blockIdx.x] = m;
    }
  }
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
  if (a.flags_self_reset && !rr && threadIdx.x == 0 && active && my_a1 > my_a0) {
    // Flags that no later kernel clears: only the last unit of this CTA's
    // range can continue on later CTAs, whose flags this CTA consumed (or
    // gave up on, which leaves the call failed and the workspace to be
    // initialised again).  Each of those CTAs sets its flag once per launch.
    const long long u_last = (my_a1 - 1) / ksteps;
    const long long u_begin = u_last * ksteps, u_end = u_begin + ksteps;
    if (u_begin >= my_a0 && u_end > my_a1) {
      const int last = atom_owner(u_end - 1, W, G);
      for (int c2 = blockIdx.x + 1; c2 <= last; ++c2) a.flags[c2] = 0;
    }
  }
  if constexpr (FP8 && C::kDual) {
    if (a.amax_n > 0) requant_tail(a, red, abort_flag);   // red / abort_flag reused as smem words
  }
}

template <Orient O, Proj P, bool FP8, int KA, int BNT>
static cudaError_t launch_one(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a,
                              int grid, cudaStream_t st) {
  using C = Cfg<O, P, FP8, KA, BNT>;
  auto kern = grouped_gemm_kernel<O, P, FP8, KA, BNT>;
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), C::kSmemBytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, st, tw, tx, a);
}

// Swap-AB pipeline shape: K atoms per stage (MOE_SWAP_KA=1|2, read once).
static int swap_ka() {
  static int v = 0;
  if (v == 0) {
    const char* s = std::getenv("MOE_SWAP_KA");
    v = (s && std::atoi(s) == 2) ? 2 : 1;
  }
  return v;
}

int gemm_swap_chunk() { return swap_ka() == 2 ? 32 : 64; }

template <Proj P, bool FP8>
static cudaError_t launch_swap(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a,
                               int grid, cudaStream_t st) {
  if (gemm_swap_chunk() == 64) return launch_one<Orient::kSwap, P, FP8, 1, 64>(tw, tx, a, grid, st);
  if (a.katoms % 2 == 0) return launch_one<Orient::kSwap, P, FP8, 2, 32>(tw, tx, a, grid, st);
  return launch_one<Orient::kSwap, P, FP8, 1, 32>(tw, tx, a, grid, st);
}

cudaError_t launch_gemm(Orient o, Proj p, bool fp8, const CUtensorMap& tw, const CUtensorMap& tx,
                        const GemmArgs& a, int grid, cudaStream_t st) {
  if (o == Orient::kSwap) {
    if (p == Proj::kW13)
      return fp8 ? launch_swap<Proj::kW13, true>(tw, tx, a, grid, st)
                 : launch_swap<Proj::kW13, false>(tw, tx, a, grid, st);
    return fp8 ? launch_swap<Proj::kW2, true>(tw, tx, a, grid, st)
               : launch_swap<Proj::kW2, false>(tw, tx, a, grid, st);
  }
  if (p == Proj::kW13)
    return fp8 ? launch_one<Orient::kNormal, Proj::kW13, true, 1, 0>(tw, tx, a, grid, st)
               : launch_one<Orient::kNormal, Proj::kW13, false, 1, 0>(tw, tx, a, grid, st);
  if (gemm_w2_pair())
    return fp8 ? launch_one<Orient::kNormal, Proj::kW2, true, 1, kPairTokens>(tw, tx, a, grid, st)
               : launch_one<Orient::kNormal, Proj::kW2, false, 1, kPairTokens>(tw, tx, a, grid, st);
  return fp8 ? launch_one<Orient::kNormal, Proj::kW2, true, 1, 0>(tw, tx, a, grid, st)
             : launch_one<Orient::kNormal, Proj::kW2, false, 1, 0>(tw, tx, a, grid, st);
}

// Normal-orientation down GEMM on 256-token chunks (two M tiles per staged
// weight tile, 128 FLOP per staged byte) unless MOE_W2_PAIR=0 (128-token
// tiles, two TMEM buffers; for measurements).
bool gemm_w2_pair() {
  static int v = -1;
  if (v < 0) {
    const char* s = std::getenv("MOE_W2_PAIR");
    v = (s && std::atoi(s) == 0) ? 0 : 1;
  }
  return v == 1;
}

int gemm_token_box_rows(Orient o) { return o == Orient::kSwap ? kTokenBox : kNormalTokens; }

int gemm_weight_box_rows(Orient o, Proj p) {
  if (o == Orient::kSwap) return kTileM;
  return p == Proj::kW13 ? 128 : 256;
}

}  // namespace moe
