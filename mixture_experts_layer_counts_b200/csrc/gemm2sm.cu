// Expert GEMMs of prefill-sized batches (normal orientation, bf16) on CTA
// pairs: one tcgen05 MMA spans the tensor cores of two SMs (cta_group::2).
//
// Why.  The single-CTA normal-orientation kernel (gemm.cu) holds a 256-token
// x 256-weight-row accumulator in one SM's TMEM (all 512 columns) and stages
// 64 KB of operands per 64-element K atom (two token tiles, 256 weight rows).
// Its ring of three such stages cannot cover the latency of weight lines that
// miss L2, so the tensor pipe idles about a third of the time.  A pair of CTAs
// computes a 256-token x 512-weight-row tile with M = 256, N = 256 MMAs whose
// A operand (tokens) is split by rows between the two SMs and whose B operand
// (weight rows) is split by rows too: each CTA stages 128 token rows and two
// 128-row weight tiles, 48 KB per K atom for the same MMA work per SM, so
// four stages fit and 25 % fewer bytes cross from L2 per multiply-add.
//   Gate/up (kW2 = false): the two weight tiles are rows [128 r, +128) of the
//   gate and of the up part of a 256-row slice of I; accumulator columns
//   [0, 256) gate, [256, 512) up; the epilogue writes h = SiLU(g) u (bf16).
//   Down (kW2 = true): the epilogue writes the router-weighted fp32 rows to
//   the assignment's slot row of ysc, as the one-CTA down GEMM does.  Its K
//   loop is short (I / 64 atoms) and its epilogue heavy, so by default
//   (kDB) a pair tile is 256 tokens x 256 rows of H, one weight tile of
//   rows [128 r, +128) per CTA and stage (six 32 KB stages), in two
//   256-column accumulators: a unit's epilogue overlaps the next unit's
//   MMAs (measured 570-594 us against 603-613 us for the 512-row form at
//   prefill-zipf; MOE_W2_2SM_DB=0 selects that form: rows [128 r, +128) of
//   each 256-row half of a 512-row slice, one 512-column accumulator).
//
// Unit = (expert, weight slice, 256-token chunk), dealt round-robin over the
// pairs in the grouped order of unit_coords (expert, then weight slice, then
// chunk), so the chunks sharing a weight slice run together.  CTA rank r of
// the pair owns token rows [128 r, 128 r + 128) of the chunk.
//
// Roles in each CTA: warp 0 lane 0 TMA producer, warp 1 TMEM allocation (both
// CTAs) and MMA issue (rank 0 only), warps 2..9 epilogue (two per TMEM lane
// quadrant, each half of the accumulator columns).
// Barriers (same shared-memory offsets in both CTAs):
//   full[s]   rank 0's: one arrival (rank 0's producer, expecting the bytes of
//             both CTAs' copies, which all complete on rank 0's barrier);
//   empty[s]  each CTA's own: released by rank 0's MMA commit (one commit per
//             CTA's barrier);
//   acc_full  each CTA's own: rank 0 commits after the unit's last K atom;
//   acc_empty rank 0's: one arrival per epilogue warp of both CTAs.
// The producers' arrivals stay inside the CTA: rank 0 alone arms full[s]
// with the bytes of both CTAs' copies (a cluster-scope release on every
// stage, as in a two-arrival form, cost about a microsecond per stage and
// left the ring serialised).
// Every wait is bounded (wait_cluster, mbar_wait): a CTA that gives up
// raises its abort flag and leaves its loops (rank 0's MMA issuer first
// waits, again bounded, for the MMAs it has in flight; copies in flight land
// within microseconds, long before a wait gives up), and both CTAs meet at
// the final cluster barrier before TMEM is released.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>

#include "common.cuh"
#include "gemm_dev.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kP2Tok = 128;                   // token rows per CTA
constexpr int kP2Rows = 128;                  // gate (and up) weight rows per CTA
constexpr int kP2Tile = 128 * kAtomBytes;     // 16 KB: one 128-row operand tile of a K atom
constexpr int kP2EpiWarps = 8;
constexpr int kP2Threads = 64 + 32 * kP2EpiWarps;
constexpr int kP2EpiLd = 20;                  // staged 32 x 16 block, rows padded to 20 words
constexpr int kP2EpiBytes = kP2EpiWarps * 32 * kP2EpiLd * 4;

// Per form: kB weight tiles per stage (two: gate and up, or two halves of
// H; one: the down GEMM's 256-row slice of H), the ring depth, and the
// accumulator buffers (one of 512 columns, or two of 256 so the epilogue of
// a unit overlaps the next unit's MMAs).
template <bool kW2, bool kDB>
struct P2 {
  static constexpr int kB = kDB ? 1 : 2;
  static constexpr int kStage = (1 + kB) * kP2Tile;
  static constexpr int kStages = kDB ? 6 : 4;
  static constexpr int kBufs = kDB ? 2 : 1;
  static constexpr int kAccCols = kB * 2 * kP2Rows;               // per buffer
  static constexpr int kSlice = kW2 ? kB * 2 * kP2Rows : 2 * kP2Rows;   // weight rows of a unit's slice
  static constexpr int kSmem = kStages * kStage + 1024 /*align*/ + 256 /*barriers*/ + kP2EpiBytes;
  static_assert(kSmem <= 232448, "shared memory");
  static_assert(!kDB || kW2, "the double-buffered form is the down GEMM's");
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_u32(p)), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Bounded wait with cluster-scope acquire (arrivals come from the other CTA too).
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status,
                                             uint32_t where, unsigned long long timeout_ns) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (try_once()) return true;
    if ((it & 31u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        report_status(status, MOE_DEVICE_TIMEOUT, where);
        *abort = 1;
        return false;
      }
    }
  }
}
// TMA 2-D tile load into this CTA's shared memory whose completion is counted
// on an mbarrier of either CTA of the pair (bar: shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, uint32_t bar, int32_t c0,
                                                 int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier (shared::cluster address, this CTA's or the peer's)
// once every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

}  // namespace

template <bool kW2, bool kDB>
__global__ void __launch_bounds__(kP2Threads, 1)
    gemm_pair2sm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  using C = P2<kW2, kDB>;
  uint8_t* tiles = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tiles + C::kStages * C::kStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + C::kBufs;
  uint64_t* drain = acc_empty + C::kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi = reinterpret_cast<float*>(tiles + C::kStages * C::kStage + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kP2EpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  grid_dependency_wait();
  grid_dependents_launch();

  const long long nchunks = static_cast<long long>(*reinterpret_cast<const volatile uint32_t*>(a.nchunks));
  const long long nunits = nchunks * a.mtiles;
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int pid = static_cast<int>(blockIdx.x >> 1);
  const int ksteps = a.katoms;
  const Segments seg0{0, 0, ksteps, true, pid, nunits, npairs};

  // rank 0's barriers as shared::cluster addresses (rank 0 itself included)
  auto full0 = [&](int s) { return peer_addr(&full[s], 0); };
  uint32_t acc_empty0[C::kBufs];
  for (int b = 0; b < C::kBufs; ++b) acc_empty0[b] = peer_addr(&acc_empty[b], 0);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------- TMA producer --
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    Segments seg = seg0;
    int u, kb0, kb1;
    while (ok && seg.next(u, kb0, kb1)) {
      int4 ch;
      int mt;
      unit_coords<true, kPairTokens>(a, u, ch, mt);
      const int e = ch.x, p0 = ch.y;
      // gate/up: rows [128 r, +128) of the gate and of the up slice (second
      // tile up_offset further); down: rows [128 r, +128) of each 256-row
      // half of the 512-row slice of H (second tile 256 further)
      const int grow = e * a.w_rows_per_expert + mt * C::kSlice + static_cast<int>(rank) * kP2Rows;
      const int second = kW2 ? 2 * kP2Rows : a.up_offset;
      const int trow = p0 + static_cast<int>(rank) * kP2Tok;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.hdr, kSiteProducerEmpty, a.timeout_ns)) {
          ok = false;
          break;
        }
        const uint32_t fb = full0(stage);
        // rank 0 expects both CTAs' bytes; rank 1's copies may land first
        // (the transaction count goes below zero until rank 0 arrives)
        if (lead) mbar_arrive_expect_tx(&full[stage], 2 * C::kStage);
        uint8_t* st = tiles + stage * C::kStage;
        const int kc = kb * 64;
        tma_load_2d_pair(st, &tm_x, fb, kc, trow, pol_x);
        tma_load_2d_pair(st + kP2Tile, &tm_w, fb, kc, grow, pol_w);
        if constexpr (C::kB == 2) tma_load_2d_pair(st + 2 * kP2Tile, &tm_w, fb, kc, grow + second, pol_w);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1 && lane == 0 && lead) {
    // ------------------------------------------------ MMA issuer (rank 0) --
    const uint32_t idesc = idesc_f32acc(1u, 2 * kP2Tok, 2 * kP2Rows);   // M = 256, N = 256, bf16
    uint32_t empty_bar[C::kStages][2];
    for (int s = 0; s < C::kStages; ++s) {
      empty_bar[s][0] = peer_addr(&empty[s], 0);
      empty_bar[s][1] = peer_addr(&empty[s], 1);
    }
    uint32_t accf[C::kBufs][2];
    for (int b = 0; b < C::kBufs; ++b) {
      accf[b][0] = peer_addr(&acc_full[b], 0);
      accf[b][1] = peer_addr(&acc_full[b], 1);
    }
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true, issued = false;
    Segments seg = seg0;
    int u, kb0, kb1;
    while (ok && seg.next(u, kb0, kb1)) {
      const int buf = it % C::kBufs;
      if (!wait_cluster(&acc_empty[buf], ((it / C::kBufs) & 1) ^ 1u, abort_flag, a.hdr, kSiteMmaAccEmpty,
                        a.timeout_ns)) {
        ok = false;
        break;
      }
      ++it;
      const uint32_t d0 = tmem_base + buf * C::kAccCols;
      tc_fence_after();
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, a.hdr, kSiteMmaFull, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(tiles + stage * C::kStage);
#pragma unroll
        for (int kk = 0; kk < kAtomBytes / 32; ++kk) {
          const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
          const uint32_t off = kk * 32;
          mma_pair(d0, sdesc_sw128(st + off), sdesc_sw128(st + kP2Tile + off), idesc, acc);
          if constexpr (C::kB == 2)
            mma_pair(d0 + 2 * kP2Rows, sdesc_sw128(st + off), sdesc_sw128(st + 2 * kP2Tile + off), idesc, acc);
        }
        issued = true;
        commit_pair(empty_bar[stage][0]);
        commit_pair(empty_bar[stage][1]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        commit_pair(accf[buf][0]);
        commit_pair(accf[buf][1]);
      }
    }
    if (!ok && issued) {
      int dummy = 0;
      commit_pair(peer_addr(drain, 0));
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy), a.hdr, kSiteDrainMma, a.timeout_ns);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue --
    // this CTA's 128 token rows; warp half hx takes half of the accumulator
    // columns.  Gate/up: h[token, i] = SiLU(g) * u over the 256-row slice of I
    // (gate at columns [0, 256), up at [256, 512)), bf16 rows of `inter`.
    // Down: the 512 columns of the H slice times the router weight, fp32 rows
    // to the assignment's slot row f of ysc (streaming stores).
    const int q = warp & 3;
    const int hx = (warp - 2) >> 2;
    float* sw = epi + (warp - 2) * 32 * kP2EpiLd;
    uint32_t* su = reinterpret_cast<uint32_t*>(sw);
    int it = 0;
    Segments seg = seg0;
    int u, kb0, kb1;
    while (seg.next(u, kb0, kb1)) {
      const int buf = it % C::kBufs;
      if (!wait_cluster(&acc_full[buf], (it / C::kBufs) & 1, abort_flag, a.hdr, kSiteEpiAccFull, a.timeout_ns)) break;
      ++it;
      tc_fence_after();
      int4 ch;
      int mt;
      unit_coords<true, kPairTokens>(a, u, ch, mt);
      const int p0 = ch.y, nv = ch.z;
      const int rb = static_cast<int>(rank) * kP2Tok + q * 32;   // first chunk row of this warp's block
      const uint32_t th = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      if constexpr (!kW2) {
        const int i0 = mt * 2 * kP2Rows;
        for (int c0 = hx * kP2Rows; c0 < (rb < nv ? (hx + 1) * kP2Rows : 0); c0 += 16) {
          float v[2][16];
          tmem_ld16x2_wait(th + c0, th + 2 * kP2Rows + c0, v[0], v[1]);
          float h[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) h[j] = __fdividef(v[0][j], 1.0f + __expf(-v[0][j])) * v[1][j];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t w4[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(h[8 * j + 2 * m], h[8 * j + 2 * m + 1]);
              w4[m] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(su + lane * kP2EpiLd + 4 * j) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          __syncwarp();
          // 2 lanes per row (32 B), 16 rows per instruction
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 16) {
            const int r = r0 + (lane >> 1);
            const uint4 val = *reinterpret_cast<const uint4*>(su + r * kP2EpiLd + 4 * (lane & 1));
            if (rb + r < nv)
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                        static_cast<size_t>(p0 + rb + r) * a.ld_out + i0 + c0 + 8 * (lane & 1)) = val;
          }
          __syncwarp();
        }
      } else {
        const int f = rb + lane < nv ? a.perm[p0 + rb + lane] : -1;
        const bool valid = f >= 0 && f < a.num_assign;
        const float wt = valid ? a.topk_w[f] : 0.f;
        const int h0 = mt * C::kSlice;
        constexpr int kHalf = C::kAccCols / 2;   // columns per warp half
        for (int c0 = hx * kHalf; c0 < (rb < nv ? (hx + 1) * kHalf : 0); c0 += 16) {
          float v[16];
          tmem_ld16_wait(th + c0, v);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4*>(sw + lane * kP2EpiLd + 4 * j) =
                make_float4(v[4 * j] * wt, v[4 * j + 1] * wt, v[4 * j + 2] * wt, v[4 * j + 3] * wt);
          __syncwarp();
          // 4 lanes per row (64 B), 8 rows per instruction
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 8) {
            const int r = r0 + (lane >> 2);
            const int fr = __shfl_sync(0xffffffffu, f, r);
            const float4 val = *reinterpret_cast<const float4*>(sw + r * kP2EpiLd + 4 * (lane & 3));
            if (fr >= 0 && fr < a.num_assign)
              __stcs(reinterpret_cast<float4*>(static_cast<float*>(a.out) + static_cast<size_t>(fr) * a.ld_out +
                                               h0 + c0 + 4 * (lane & 3)), val);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cluster(acc_empty0[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no MMA, copy or arrival of either CTA is still pending on the other
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

static int env_on(const char* name) {
  const char* s = std::getenv(name);
  return (s && std::atoi(s) == 0) ? 0 : 1;
}

bool w13_pair2sm_supported(int I, bool fp8) {
  static const int v = env_on("MOE_W13_2SM");
  return v == 1 && !fp8 && I % (2 * kP2Rows) == 0;
}

bool w2_pair2sm_supported(int H, bool fp8) {
  static const int v = env_on("MOE_W2_2SM");
  return v == 1 && !fp8 && H % (4 * kP2Rows) == 0;
}

template <bool kW2, bool kDB>
static cudaError_t launch_pair2sm(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int max_ctas,
                                  cudaStream_t st) {
  using C = P2<kW2, kDB>;
  auto kern = gemm_pair2sm_kernel<kW2, kDB>;
  cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), C::kSmem);
  if (err != cudaSuccess) return err;
  // as many CTA pairs as can be resident at once (one CTA per SM)
  static int pairs_cache[64] = {0};   // per device (and per form: one instance per template)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  int pairs = (dev >= 0 && dev < 64) ? pairs_cache[dev] : 0;
  if (pairs == 0) {
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * (max_ctas / 2));
    q.blockDim = dim3(kP2Threads);
    q.dynamicSmemBytes = C::kSmem;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, kern, &q);
    if (err != cudaSuccess) return err;
    pairs = n < 1 ? 1 : n;
    if (dev >= 0 && dev < 64) pairs_cache[dev] = pairs;
  }
  if (pairs > max_ctas / 2) pairs = max_ctas / 2 > 0 ? max_ctas / 2 : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kP2Threads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  GemmArgs g = a;
  // slices per CTA pair: 256 rows of I (gate/up) or C::kSlice rows of H (down)
  g.mtiles = kW2 ? a.w_rows_per_expert / C::kSlice : a.up_offset / C::kSlice;
  return cudaLaunchKernelEx(&cfg, kern, tw, tx, g);
}

cudaError_t launch_w13_pair2sm(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int max_ctas,
                               cudaStream_t st) {
  return launch_pair2sm<false, false>(tw, tx, a, max_ctas, st);
}

cudaError_t launch_w2_pair2sm(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int max_ctas,
                              cudaStream_t st) {
  static const int db = env_on("MOE_W2_2SM_DB");
  if (db) return launch_pair2sm<true, true>(tw, tx, a, max_ctas, st);
  return launch_pair2sm<true, false>(tw, tx, a, max_ctas, st);
}

}  // namespace moe
