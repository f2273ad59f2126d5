// Fused expert FFN of decode batches: the gate/up GEMM (SiLU * up epilogue)
// and the down GEMM (router-weighted slot rows) in one persistent launch,
// swap-AB orientation, bf16.
//
// Why.  At decode every active expert's weights are streamed once and the
// layer is bound by HBM; between two launches the first GEMM's tail (CTAs
// finishing at different times) and the second's ramp (launch, prologue,
// pipeline fill) leave HBM partly idle.  Here each CTA streams its share of
// the gate/up weights and then, without a launch boundary, its share of the
// down weights.
//
// Work split.  Both GEMMs use the stream-K split of the grouped kernels: the
// units (token chunk x 128-row weight tile) x K steps of each GEMM are cut
// into G equal contiguous ranges in chunk-major order, one per CTA; a unit cut
// by a range boundary is finished by its head CTA from the others' fp32
// partial tiles (gemm_dev.cuh).  Because both orders are chunk-major and the
// ranges are proportional, the down-projection units of CTA c mostly belong
// to chunks whose gate/up units CTA c (or a neighbour) already finished.
//
// Dependency.  A down-projection unit of chunk c reads the intermediate rows
// of chunk c, complete once all I/128 gate/up units of the chunk have run
// their epilogue.  The epilogue of each gate/up unit publishes its rows with
// a release increment of dep[c] (after a barrier of the epilogue warps); the
// producer acquires dep[c] == I/128 (bounded wait) and orders its TMA reads
// after it with a proxy fence before it loads chunk c's intermediate rows.
// The weight tiles of that stage do not depend on it.
//
// Pipeline.  Warp 0 lane 0: TMA producer; warp 1 lane 0: MMA issuer; warps
// 2..5: epilogue (one TMEM lane quadrant each).  A stage holds one K atom of
// gate + up + tokens (gate/up GEMM) or two K atoms of weights + tokens (down
// GEMM), 40 KB, five stages; the producer's ring position, the MMA's TMEM
// buffer count and the epilogue's unit count run on across the two GEMMs.
// Token chunks hold at most 32 tokens (MMA N <= 32), so the host uses this
// kernel for calls with T <= 32 (no expert can then have more tokens).
// Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_dev.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kFfnBN = 32;                                   // largest token chunk (MMA N)
constexpr int kFfnATile = kTileM * kAtomBytes;               // 128 weight rows x 128 B
constexpr int kFfnBTile = kFfnBN * kAtomBytes;               // 32 token rows x 128 B
constexpr int kFfnStage = 2 * (kFfnATile + kFfnBTile);       // 40 KB
constexpr int kFfnStages = (232448 - 1280) / kFfnStage;
constexpr int kFfnThreads = 192;
constexpr int kFfnEpiWarps = 4;
constexpr int kFfnAccCols = 2 * kFfnBN;                      // per TMEM buffer: gate + up
constexpr int kFfnTmemCols = 2 * kFfnAccCols;                // two buffers
constexpr int kFfnSmem = kFfnStages * kFfnStage + 1024 + 256;
static_assert(kFfnStages >= 4, "pipeline depth");
static_assert(kFfnSmem <= 232448, "shared memory");

struct FfnArgs {
  GemmArgs g13, g2;
  int* dep;          // [chunks] finished gate/up units per token chunk (zero at launch)
};

__device__ __forceinline__ int ld_acquire_i(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *p >= want.
__device__ __forceinline__ bool wait_count(const int* p, int want, volatile int* abort, uint32_t* status,
                                           unsigned long long timeout_ns) {
  if (ld_acquire_i(p) >= want) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_i(p) >= want) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        report_status(status, MOE_DEVICE_TIMEOUT, kSiteDependency);
        *abort = 1;
        return false;
      }
    }
  }
}

// Stream-K range of this CTA in one GEMM: W = units * ksteps.
__device__ __forceinline__ Segments ffn_segments(long long nunits, int ksteps, bool& active, int& G,
                                                 long long& W) {
  W = nunits * ksteps;
  G = static_cast<int>(W / kMinAtomsPerCta);
  G = G < 1 ? 1 : (G > static_cast<int>(gridDim.x) ? static_cast<int>(gridDim.x) : G);
  active = W > 0 && static_cast<int>(blockIdx.x) < G;
  const long long a0 = active ? range_begin(W, G, blockIdx.x) : 0;
  const long long a1 = active ? range_begin(W, G, blockIdx.x + 1) : 0;
  return Segments{a0, a1, ksteps, false, 0, 0, 1};
}

__device__ __forceinline__ int ffn_cols(int nv) { return (nv + kTokenBox - 1) / kTokenBox * kTokenBox; }

}  // namespace

__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_swap_kernel(const __grid_constant__ CUtensorMap tm_w13, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_h,
                    const FfnArgs f) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* tiles = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tiles + kFfnStages * kFfnStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + kFfnStages;
  uint64_t* acc_full = bars + 2 * kFfnStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const GemmArgs& a1 = f.g13;
  const GemmArgs& a2 = f.g2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFfnStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * kFfnEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_w13);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w2);
    tma_prefetch_desc(&tm_h);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kFfnTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The schedule (chunks, their count) was written by the align kernel, which
  // has completed when this grid is launched (the gather kernel before it
  // starts its dependents only after its own wait).
  const long long nchunks = *reinterpret_cast<const volatile uint32_t*>(a1.nchunks);
  const int ks1 = a1.katoms;          // one K atom per stage
  const int ks2 = a2.katoms / 2;      // two K atoms per stage
  bool act1, act2;
  int G1, G2;
  long long W1, W2;
  const Segments seg1 = ffn_segments(nchunks * a1.mtiles, ks1, act1, G1, W1);
  const Segments seg2 = ffn_segments(nchunks * a2.mtiles, ks2, act2, G2, W2);

  const bool producer = warp == 0 && lane == 0;
  if (!producer) {
    grid_dependency_wait();
    grid_dependents_launch();
  }

  if (producer) {
    // ---------------------------------------------------------- TMA producer --
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    uint32_t armed = 0, armed_parity = 0;
    auto chunk_of = [&](const GemmArgs& a, int u) { return a.chunks[u / a.mtiles]; };
    // gate/up stage: parts bit 0 = gate and up tiles, bit 1 = token tiles.
    // Failure-path test: CTA 0 issues nothing for its first stage, so a
    // bounded wait runs out.
    auto issue1 = [&](int stage, int u, int kb, int parts, bool first) {
      if (a1.inject_stall != 0 && blockIdx.x == 0 && first) return;
      const int4 ch = chunk_of(a1, u);
      const int mt = u - (u / a1.mtiles) * a1.mtiles;
      const int wrow0 = ch.x * a1.w_rows_per_expert + mt * kTileM;
      uint8_t* st = tiles + stage * kFfnStage;
      const int kc = kb * 64;   // bf16 elements
      if (parts & 1) {
        tma_load_2d(st, &tm_w13, &full[stage], kc, wrow0, pol_w);
        tma_load_2d(st + kFfnATile, &tm_w13, &full[stage], kc, wrow0 + a1.up_offset, pol_w);
      }
      if (parts & 2) {
        const int nbox = ffn_cols(ch.z) / kTokenBox;
        for (int q = 0; q < nbox; ++q)
          tma_load_2d(st + 2 * kFfnATile + q * kTokenBox * kAtomBytes, &tm_x, &full[stage], kc,
                      ch.y + q * kTokenBox, pol_x);
      }
    };
    auto bytes1 = [&](int u) -> uint32_t { return 2 * kFfnATile + ffn_cols(chunk_of(a1, u).z) * kAtomBytes; };

    // (1) before the wait for the gather: arm the first stages, fetch their weights
    int pre = 0;
    if (act1) {
      Segments seg = seg1;
      int u, kb0, kb1;
      while (pre < kFfnStages && seg.next(u, kb0, kb1)) {
        const uint32_t b = bytes1(u);
        for (int kb = kb0; kb < kb1 && pre < kFfnStages; ++kb, ++pre) {
          mbar_arrive_expect_tx(&full[pre], b);
          armed |= 1u << pre;
          issue1(pre, u, kb, 1, pre == 0);
        }
      }
    }
    grid_dependency_wait();
    grid_dependents_launch();

    int stage = 0;
    uint32_t phase = 0;
    int n = 0;
    bool ok = true;
    auto advance = [&]() {
      if (++stage == kFfnStages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    // (2) gate/up GEMM
    if (act1) {
      Segments seg = seg1;
      int u, kb0, kb1;
      while (ok && seg.next(u, kb0, kb1)) {
        const uint32_t b = bytes1(u);
        for (int kb = kb0; kb < kb1; ++kb, ++n) {
          if (n < pre) {
            issue1(stage, u, kb, 2, n == 0);
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a1.hdr, kSiteProducerEmpty, a1.timeout_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], b);
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            issue1(stage, u, kb, 3, false);
          }
          advance();
        }
      }
    }
    // (3) down GEMM: two K atoms per stage; a chunk's intermediate rows are
    // loaded only after all of its gate/up units have published them
    if (act2) {
      Segments seg = seg2;
      int u, kb0, kb1;
      int ready_chunk = -1;
      while (ok && seg.next(u, kb0, kb1)) {
        const int cs = u / a2.mtiles;
        const int4 ch = a2.chunks[cs];
        const int mt = u - cs * a2.mtiles;
        const int wrow0 = ch.x * a2.w_rows_per_expert + mt * kTileM;
        const int nbox = ffn_cols(ch.z) / kTokenBox;
        const uint32_t b = 2 * (kFfnATile + ffn_cols(ch.z) * kAtomBytes);
        for (int kb = kb0; kb < kb1; ++kb, ++n) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a2.hdr, kSiteProducerEmpty, a2.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], b);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          uint8_t* st = tiles + stage * kFfnStage;
          for (int ka = 0; ka < 2; ++ka)
            tma_load_2d(st + ka * (kFfnATile + kFfnBTile), &tm_w2, &full[stage], (2 * kb + ka) * 64, wrow0, pol_w);
          if (cs != ready_chunk) {
            if (!wait_count(f.dep + cs, a1.mtiles, abort_flag, a2.hdr, a2.timeout_ns)) {
              ok = false;   // the weight copies of this stage are in flight: drained below
              break;
            }
            fence_proxy_async_global();
            ready_chunk = cs;
          }
          for (int ka = 0; ka < 2; ++ka)
            for (int q = 0; q < nbox; ++q)
              tma_load_2d(st + ka * (kFfnATile + kFfnBTile) + kFfnATile + q * kTokenBox * kAtomBytes, &tm_h,
                          &full[stage], (2 * kb + ka) * 64, ch.y + q * kTokenBox, pol_x);
          advance();
        }
      }
    }
    if (!ok) {
      // let copies already in flight land before the CTA's smem is released (a
      // stage whose token copies were never issued does not complete: its wait
      // runs out after the limit)
      int dummy = 0;
      const unsigned long long lim = a1.timeout_ns < 50000000ull ? a1.timeout_ns : 50000000ull;
      for (int s = 0; s < kFfnStages; ++s)
        if ((armed >> s) & 1u)
          mbar_wait(&full[s], (armed_parity >> s) & 1u, reinterpret_cast<volatile int*>(&dummy), a1.hdr,
                    kSiteDrainTma, lim);
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- MMA issuer --
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    bool issued = false;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const GemmArgs& a = ph == 0 ? a1 : a2;
      if (!(ph == 0 ? act1 : act2)) continue;
      Segments seg = ph == 0 ? seg1 : seg2;
      int u, kb0, kb1;
      while (ok && seg.next(u, kb0, kb1)) {
        const int buf = it & 1;
        const uint32_t accph = (it >> 1) & 1;
        ++it;
        if (!mbar_wait(&acc_empty[buf], accph ^ 1u, abort_flag, a.hdr, kSiteMmaAccEmpty, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int4 ch = a.chunks[u / a.mtiles];
        const uint32_t idesc = idesc_f32acc(1u, kTileM, static_cast<uint32_t>(ffn_cols(ch.z)));
        const uint32_t d0 = tmem_base + buf * kFfnAccCols;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, a.hdr, kSiteMmaFull, a.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * kFfnStage);
          if (ph == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
              const uint32_t sb = st + 2 * kFfnATile + kk * 32;
              mma_ss<false>(d0, sdesc_sw128(st + kk * 32), sdesc_sw128(sb), idesc, acc);
              mma_ss<false>(d0 + kFfnBN, sdesc_sw128(st + kFfnATile + kk * 32), sdesc_sw128(sb), idesc, acc);
            }
          } else {
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) {
              const int ka = kq >> 2, kk = kq & 3;
              const uint32_t sa = st + ka * (kFfnATile + kFfnBTile);
              const uint32_t acc = (kb > kb0 || kq > 0) ? 1u : 0u;
              mma_ss<false>(d0, sdesc_sw128(sa + kk * 32), sdesc_sw128(sa + kFfnATile + kk * 32), idesc, acc);
            }
          }
          issued = true;
          mma_commit(&empty[stage]);
          if (++stage == kFfnStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
    }
    if (!ok && issued) {
      int dummy = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), a1.hdr, kSiteDrainMma, a1.timeout_ns);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue --
    constexpr int kEpiThreads = 32 * kFfnEpiWarps;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;   // 0 .. kEpiThreads - 1
    int it = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const GemmArgs& a = ph == 0 ? a1 : a2;
      if (!(ph == 0 ? act1 : act2)) continue;
      const long long W = ph == 0 ? W1 : W2;
      const int G = ph == 0 ? G1 : G2;
      const int ksteps = ph == 0 ? ks1 : ks2;
      Segments seg = ph == 0 ? seg1 : seg2;
      int u, kb0, kb1;
      while (seg.next(u, kb0, kb1)) {
        const int buf = it & 1;
        const uint32_t accph = (it >> 1) & 1;
        ++it;
        if (!mbar_wait(&acc_full[buf], accph, abort_flag, a.hdr, kSiteEpiAccFull, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int cs = u / a.mtiles;
        const int4 ch = a.chunks[cs];
        const int mt = u - cs * a.mtiles;
        const int p0 = ch.y, nv = ch.z;
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kFfnAccCols;
        const int ncols = ffn_cols(nv);
        const int nacc = ph == 0 ? 2 : 1;

        if (kb0 > 0) {
          // later piece of a split unit: hand the raw accumulator(s) over
          float* slot = a.partials + static_cast<size_t>(blockIdx.x) * kPartialSlotFloats;
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float v[2][16];
            if (nacc == 2)
              tmem_ld16x2_wait(tbase + c0, tbase + kFfnBN + c0, v[0], v[1]);
            else
              tmem_ld16_wait(tbase + c0, v[0]);
            for (int ac = 0; ac < nacc; ++ac) {
              float4* dst = reinterpret_cast<float4*>(slot + (static_cast<size_t>(ac) * kTileM + row) * kFfnBN + c0);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                __stcg(dst + j, make_float4(v[ac][4 * j], v[ac][4 * j + 1], v[ac][4 * j + 2], v[ac][4 * j + 3]));
            }
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          __threadfence();
          epilogue_bar<kEpiThreads>();
          if (row == 0) st_release(a.flags + blockIdx.x, 1);
          continue;
        }

        // first atoms of the unit: collect the later pieces, then finish
        int last = blockIdx.x;
        if (kb1 < ksteps) {
          const long long unit_end = (static_cast<long long>(u) + 1) * ksteps;
          last = atom_owner(unit_end - 1, W, G);
          bool fl = true;
          for (int c2 = blockIdx.x + 1; c2 <= last && fl; ++c2)
            fl = wait_flag(a.flags + c2, abort_flag, a.hdr, a.timeout_ns);
          if (!fl) {
            ok = false;
            break;
          }
        }
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[2][16];
          if (nacc == 2)
            tmem_ld16x2_wait(tbase + c0, tbase + kFfnBN + c0, v[0], v[1]);
          else
            tmem_ld16_wait(tbase + c0, v[0]);
          for (int c2 = blockIdx.x + 1; c2 <= last; ++c2) {
            const float* slot = a.partials + static_cast<size_t>(c2) * kPartialSlotFloats;
            for (int ac = 0; ac < nacc; ++ac) {
              const float4* src =
                  reinterpret_cast<const float4*>(slot + (static_cast<size_t>(ac) * kTileM + row) * kFfnBN + c0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 pv = __ldcg(src + j);
                v[ac][4 * j] += pv.x;
                v[ac][4 * j + 1] += pv.y;
                v[ac][4 * j + 2] += pv.z;
                v[ac][4 * j + 3] += pv.w;
              }
            }
          }
          if (ph == 0) {
            // h = SiLU(g) * u, rounded once to bf16, row = intermediate column
            const int irow = mt * kTileM + row;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int nn = c0 + j;
              if (nn < nv) {
                const float gg = v[0][j], uv = v[1][j];
                const float h = __fdividef(gg, 1.0f + __expf(-gg)) * uv;
                static_cast<__nv_bfloat16*>(a.out)[static_cast<size_t>(p0 + nn) * a.ld_out + irow] =
                    __float2bfloat16_rn(h);
              }
            }
          } else {
            // router-weighted fp32 slot rows, row = hidden index
            const int hrow = mt * kTileM + row;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int nn = c0 + j;
              const int fl = nn < nv ? a.perm[p0 + nn] : -1;
              if (fl >= 0 && fl < a.num_assign)
                static_cast<float*>(a.out)[static_cast<size_t>(fl) * a.ld_out + hrow] = v[0][j] * a.topk_w[fl];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);

        if (ph == 0) {
          // publish the unit's intermediate rows: every epilogue store
          // precedes the barrier; one release increment of the chunk's count
          epilogue_bar<kEpiThreads>();
          if (et == 0) red_release_add(f.dep + cs, 1);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kFfnTmemCols);
}

bool ffn_swap_supported(int T, int H, int I) {
  // chunks of at most 32 tokens (T <= 32 guarantees it); both K extents whole stages
  return T <= kFfnBN && H % 128 == 0 && I % 128 == 0;
}

int ffn_swap_chunk() { return kFfnBN; }

cudaError_t launch_ffn_swap(const CUtensorMap& tw13, const CUtensorMap& tx, const CUtensorMap& tw2,
                            const CUtensorMap& th, const GemmArgs& g13, const GemmArgs& g2, int* dep, int grid,
                            cudaStream_t st) {
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(ffn_swap_kernel), kFfnSmem);
  if (err != cudaSuccess) return err;
  FfnArgs f{g13, g2, dep};
  return launch_pdl(ffn_swap_kernel, dim3(grid), dim3(kFfnThreads), kFfnSmem, st, tw13, tx, tw2, th, f);
}

}  // namespace moe
