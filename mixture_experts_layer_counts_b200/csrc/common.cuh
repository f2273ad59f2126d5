// Shared definitions of the fused-MoE CUDA library: status codes, tile
// constants, the workspace layout and the device-side status word.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace moe {

// Device status codes (same values as moe_status_t in include/moe.h).
constexpr uint32_t MOE_DEVICE_OK = 0;
constexpr uint32_t MOE_DEVICE_TIMEOUT = 5;
constexpr uint32_t MOE_DEVICE_BOUNDS = 6;

// Where a device wait gave up (low byte of the status info word).
enum WaitSite : uint32_t {
  kSiteProducerEmpty = 1,
  kSiteMmaFull = 2,
  kSiteMmaAccEmpty = 3,
  kSiteEpiAccFull = 4,
  kSiteDrainTma = 5,
  kSiteDrainMma = 6,
  kSiteGridBarrier = 7,
  kSiteDependency = 8,     // fused FFN: a down-projection tile waited for its gate/up rows
};

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s per wait

// Tile geometry.  One K atom is 128 bytes of a row: 64 bf16 or 128 E4M3.
constexpr int kAtomBytes = 128;
constexpr int kTileM = 128;            // rows of the A operand per MMA (M)
constexpr int kSwapMaxTokens = 64;     // largest token chunk in swap-AB (N <= 64)
constexpr int kTokenBox = 16;          // rows per TMA box of the token operand (swap-AB)
constexpr int kNormalTokens = 128;     // token rows per tile in normal orientation (M)
constexpr int kPairTokens = 256;       // gate/up GEMM, normal orientation: two M tiles per weight tile
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kMaxGrid = 1024;          // persistent grids never exceed this
constexpr int kMaxSlots = 160;          // GEMM CTAs per launch (>= the SM count of a B200)
constexpr int kPartialSlotFloats = 32768;   // fp32 partial tile of one GEMM CTA (128 KB)
constexpr int kGemmLaunches = 4;        // {w13, w2} x {swap-AB, normal}: one flag array each

// Header words at the start of the workspace (uint32 units).
constexpr int kHdrStatus = 0;          // first device error code (sticky)
constexpr int kHdrInfo = 1;            // where it happened
constexpr int kHdrChunksSwap = 4;      // number of swap-AB token chunks
constexpr int kHdrChunksNormal = 5;    // number of normal-orientation token tiles
constexpr int kHdrUncertain = 6;       // tokens whose router ordering needed fp64 / exact
constexpr int kHdrChunksPair = 7;      // number of normal-orientation 256-token chunks (gate/up GEMM)
constexpr int kHdrScaleS1 = 8;         // fp32 bits: activation scale (FP8)
constexpr int kHdrScaleS2 = 9;         // fp32 bits: intermediate scale (FP8)
constexpr int kHdrBarrier = 12;        // grid barrier counter
constexpr int kHdrRouterAll = 13;      // top-k CTAs finished (decode calls: the last one aligns;
                                       // reset by that CTA, so every call starts at 0)
constexpr int kHdrRouterFlags = 64;    // words 64 .. 64 + kMaxSlots - 1: split-unit flags of the
                                       // tensor-core router GEMM (zeroed again by their consumer)
constexpr int kHeaderBytes = 1024;
constexpr int kStatusBytes = kHeaderBytes;

__device__ __forceinline__ void report_status(uint32_t* status, uint32_t code, uint32_t where) {
  if (atomicCAS(status + kHdrStatus, 0u, code) == 0u) {
    atomicExch(status + kHdrInfo, where);
  }
}

// Byte offsets of every region of the caller-provided workspace.
struct Layout {
  size_t header, topk_ids, topk_w, logits, xnorm, wnorm, amax_tok, amax_cta, cand, rsplit;
  size_t slice_hist;
  size_t counts, offsets, perm, inv_perm, chunks_swap, chunks_normal, chunks_pair, gemm_flags, partials;
  size_t partials2;            // second set of partial tiles (the fused FFN's down GEMM)
  int n_gemm_flags;            // split-tile flags of every GEMM launch + per-chunk counters
  size_t xperm, inter, h32, ysc, staging_in, staging_out, total;
  int max_chunks_swap, max_chunks_normal, max_chunks_pair;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Split-K router partials: up to kRouterSplits partial logit matrices and
// partial sums for the norms and amax (see the tiled logits kernel).
constexpr int kRouterSplits = 4;
// moe_align: T*k at or above kAlignSliceMin runs as two grids over at most
// kAlignMaxSlices slices (per-slice expert counts in the workspace).
constexpr int kAlignSliceMin = 8192;
constexpr int kAlignMaxSlices = 256;
inline size_t router_split_floats(int T, int E) {
  return static_cast<size_t>(kRouterSplits) * (static_cast<size_t>(T) * E + 2 * static_cast<size_t>(T) + E);
}

inline Layout make_layout(int T, int H, int E, int I, int k, bool fp8) {
  Layout L{};
  size_t A = static_cast<size_t>(T) * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.header = take(kHeaderBytes);
  L.topk_ids = take(A * 4);
  L.topk_w = take(A * 4);
  L.logits = take(static_cast<size_t>(T) * E * 4);
  L.xnorm = take(static_cast<size_t>(T) * 4);
  L.wnorm = take(static_cast<size_t>(E) * 4);
  L.amax_tok = take(static_cast<size_t>(T) * 4);
  L.amax_cta = take(static_cast<size_t>(kMaxGrid) * 4);
  L.cand = take(static_cast<size_t>(T) * E * 16);    // router fallback scratch
  L.rsplit = take(router_split_floats(T, E) * 4);     // split-K router partials
  L.counts = take(static_cast<size_t>(E) * 4);
  L.offsets = take(static_cast<size_t>(E + 1) * 4);
  L.perm = take(A * 4);
  L.inv_perm = take(A * 4);
  L.slice_hist = take(static_cast<size_t>(kAlignMaxSlices) * E * 4);
  L.max_chunks_swap = static_cast<int>(E + A / 16 + 1);   // swap chunks hold >= 16 tokens
  L.max_chunks_normal = static_cast<int>(E + A / kNormalTokens + 1);
  L.chunks_swap = take(static_cast<size_t>(L.max_chunks_swap) * 16);
  L.chunks_normal = take(static_cast<size_t>(L.max_chunks_normal) * 16);
  L.max_chunks_pair = static_cast<int>(E + A / kPairTokens + 1);
  L.chunks_pair = take(static_cast<size_t>(L.max_chunks_pair) * 16);
  // flags of the GEMM launches, then one counter per swap-AB chunk (the fused
  // FFN's gate/up -> down dependency); all zeroed by the align kernel
  L.n_gemm_flags = kGemmLaunches * kMaxSlots + L.max_chunks_swap;
  L.gemm_flags = take(static_cast<size_t>(L.n_gemm_flags) * 4);
  L.partials = take(static_cast<size_t>(kMaxSlots) * kPartialSlotFloats * 4);
  L.partials2 = take(static_cast<size_t>(kMaxSlots) * kPartialSlotFloats * 4);
  const size_t eb = fp8 ? 1 : 2;
  L.xperm = take(A * H * eb);
  L.inter = take(A * I * eb);
  L.h32 = fp8 ? take(A * I * 4) : off;
  L.ysc = take(A * H * 4);
  L.staging_in = take(static_cast<size_t>(T) * H * 2);
  L.staging_out = take(static_cast<size_t>(T) * H * 2);
  L.total = off;
  return L;
}

}  // namespace moe
