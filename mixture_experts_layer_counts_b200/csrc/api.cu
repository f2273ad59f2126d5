// C ABI of the fused MoE layer: argument checks, workspace carve-up,
// per-expert orientation policy, tensor maps and the launch sequence.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

cudaError_t set_smem_limit_once(const void* kernel, int bytes) {
  struct Entry {
    const void* kernel;
    int device;
    int bytes;
  };
  static std::mutex mu;
  static Entry table[256];
  static int n = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (table[i].kernel == kernel && table[i].device == dev && table[i].bytes >= bytes) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return err;
  for (int i = 0; i < n; ++i)
    if (table[i].kernel == kernel && table[i].device == dev) {
      table[i].bytes = bytes;
      return cudaSuccess;
    }
  if (n < 256) table[n++] = Entry{kernel, dev, bytes};
  return cudaSuccess;
}

int current_sm_count() {
  constexpr int kDevices = 64;
  static int cache[kDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

namespace {

constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int device_sm_count() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// Experts with at most this many tokens run swap-AB (weights in M, tokens in
// N); heavier experts run the normal orientation.  MOE_SWAP_MAX_TOKENS
// overrides it (for measurements), clamped to [0, kSwapMaxTokens].
int swap_threshold() {
  static int v = -1;
  if (v < 0) {
    const char* s = std::getenv("MOE_SWAP_MAX_TOKENS");
    int t = s ? std::atoi(s) : kSwapMaxTokens;
    v = t < 0 ? 0 : (t > kSwapMaxTokens ? kSwapMaxTokens : t);
  }
  return v;
}

// The fused decode FFN launch is on by default; MOE_FUSED_FFN=0 selects the
// two-launch path (for measurements).
bool fused_ffn_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* s = std::getenv("MOE_FUSED_FFN");
    v = (s && std::atoi(s) == 0) ? 0 : 1;
  }
  return v == 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_shape(int T, int H, int E, int I, int k, int dtype) {
  if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (k < 1 || k > E || k > kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (T < 1 || static_cast<long long>(T) * k > (1LL << 24)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (H < 128 || H > 8192 || H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (I < 128 || I > 16384 || I % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status_t make_tmap(CUtensorMap* m, const void* base, bool fp8, int inner, long long rows,
                       int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return MOE_ERR_CUDA;
  const int esize = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kAtomBytes / esize), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                  \
  do {                                 \
    moe_status_t s_ = (expr);          \
    if (s_ != MOE_OK) return s_;       \
  } while (0)

// Stage events: inside a stream capture a plain record would only be a
// dependency marker of the graph, so record "external" event nodes there.
void record(moe_debug_out_t* dbg, int i, cudaStream_t st) {
  if (!(dbg && dbg->stage_events && dbg->stage_events[i])) return;
  cudaEvent_t ev = static_cast<cudaEvent_t>(dbg->stage_events[i]);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

// Large batches: router logits on the tensor cores (the swap-AB kernel in its
// dense router mode: expert rows in M, 64-token chunks of hidden in N, fp32
// accumulation, whole units dealt round-robin), then the top-k kernel.  The
// logits carry at most H * 2^-22 * ||x|| ||w|| of error: every MMA adds 16
// exact bf16 products to the fp32 accumulator, and even an accumulation that
// aligns them to the largest exponent and truncates loses at most 17 units in
// the last place of the running magnitude per instruction (H / 16
// instructions; a factor 2 of margin).  Tokens whose top-(k+1) gaps that
// bound cannot separate are re-ranked in fp64, then exactly, as on every path.
// Router path: logits on the tensor cores (route_tc) once the logit work
// passes 2^28 multiply-adds (large batches, where the CUDA-core kernels are
// bound by their arithmetic), else the CUDA-core logits kernels, whose
// tighter bounds certify most tokens without a second pass.  MOE_ROUTER=tc or
// =simt fixes the path for calls that need not be batch-invariant (for
// measurements and tests).
bool tc_router_eligible(int T, int H, int E, bool invariant) {
  static int force = -1;   // 0: size rule, 1: tensor cores, 2: CUDA cores
  if (force < 0) {
    const char* s = std::getenv("MOE_ROUTER");
    force = !s ? 0 : (std::strcmp(s, "tc") == 0 ? 1 : (std::strcmp(s, "simt") == 0 ? 2 : 0));
  }
  if (invariant || force == 2) return false;
  return force == 1 || static_cast<double>(T) * E * H > static_cast<double>(1 << 28);
}

// Logits on the tensor cores as a dense swap-AB GEMM (router rows = M, tokens
// = N), its K loop split over the grid with partial tiles when `ra.partials`
// is given (flags in the workspace header, cleared again by their consumer),
// then the candidate re-evaluation top-k (launch_router_topk_tc).
moe_status_t route_tc(const RouterArgs& ra, int grid, unsigned long long timeout_ns, cudaStream_t st,
                      const AlignArgs* fuse_align = nullptr, bool* fused = nullptr) {
  CUtensorMap tw, tx;
  MOE_TRY(make_tmap(&tw, ra.router_w, false, ra.H, ra.E, gemm_weight_box_rows(Orient::kSwap, Proj::kW2)));
  MOE_TRY(make_tmap(&tx, ra.hidden, false, ra.H, ra.T, gemm_token_box_rows(Orient::kSwap)));
  GemmArgs g{};
  g.dense_T = ra.T;
  g.dense_chunk = gemm_swap_chunk();
  g.n_cols = ra.E;
  g.col_bias = ra.bias;
  g.norm_x = ra.hidden;
  g.norm_w = ra.router_w;
  g.xnorm = ra.xnorm;
  g.wnorm = ra.wnorm;
  g.amax_tok = ra.amax_tok;
  g.norm_H = ra.H;
  g.mtiles = (ra.E + kTileM - 1) / kTileM;
  g.katoms = ra.H * 2 / kAtomBytes;
  g.w_rows_per_expert = 0;
  g.out = ra.logits;
  g.ld_out = ra.E;
  g.num_assign = ra.T;
  g.hdr = ra.hdr;
  g.timeout_ns = timeout_ns;
  g.whole_units = ra.partials != nullptr ? 0 : 1;
  g.partials = ra.partials;
  g.flags = reinterpret_cast<int*>(ra.hdr + kHdrRouterFlags);
  g.flags_self_reset = 1;
  MOE_TRY(cuda_status(launch_gemm(Orient::kSwap, Proj::kW2, false, tw, tx, g, grid, st)));
  // H 2^-22 ||x|| ||w||: the tensor-core accumulation order and rounding are
  // not specified, so the bound allows four ulps of sum|x w| per product
  const float gamma = static_cast<float>(static_cast<double>(ra.H) * 2.384185791015625e-07);
  const float ulast = 1.1920928955078125e-07f;   // the partial-tile adds, the bias add
  return cuda_status(launch_router_topk_tc(ra, gamma, ulast, st, fuse_align, fused));
}

moe_status_t forward_impl(const void* hidden, const void* router_w, const float* router_bias,
                          const void* w13, const void* w2, const float* w13_scale,
                          const float* w2_scale, int T, int H, int E, int I, int k, int dtype,
                          void* out, void* ws, size_t ws_bytes, moe_debug_out_t* dbg,
                          cudaStream_t st, bool invariant = false, bool out_fp32 = false) {
  MOE_TRY(check_shape(T, H, E, I, k, dtype));
  const bool fp8 = dtype == MOE_DTYPE_FP8_E4M3;
  if (invariant && fp8) return MOE_ERR_INVALID_ARG;   // per-tensor FP8 scales span the batch
  if (!hidden || !router_w || !w13 || !w2 || !out || !ws) return MOE_ERR_INVALID_ARG;
  if (fp8 && (!w13_scale || !w2_scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(router_w) || !aligned16(w13) || !aligned16(w2) ||
      !aligned16(out) || !aligned16(ws) || (router_bias && (reinterpret_cast<uintptr_t>(router_bias) & 3u)))
    return MOE_ERR_MISALIGNED;
  const Layout L = make_layout(T, H, E, I, k, fp8);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const int A = T * k;
  uint32_t* hdr = at<uint32_t>(ws, L.header);

  int tau = swap_threshold();
  if (dbg && (dbg->force_orient == 1 || dbg->force_orient == 3)) tau = INT_MAX;
  if (dbg && dbg->force_orient == 2) tau = 0;
  if (H % 256 != 0) tau = INT_MAX;   // the normal-orientation w2 tile is 256 rows of H
  if (invariant) tau = INT_MAX;       // one orientation for every expert and batch
  const bool any_swap = tau > 0;
  const bool any_normal = T > tau;

  // tensor maps (weights and grouped activations), built before any launch
  CUtensorMap tw13s, tw13n, tw2s, tw2n, tw2p, txs, txn, tis, tin;
  const long long w13_rows = static_cast<long long>(E) * 2 * I;
  const long long w2_rows = static_cast<long long>(E) * H;
  void* xperm = at<void>(ws, L.xperm);
  void* inter = at<void>(ws, L.inter);
  if (any_swap) {
    MOE_TRY(make_tmap(&tw13s, w13, fp8, H, w13_rows, gemm_weight_box_rows(Orient::kSwap, Proj::kW13)));
    MOE_TRY(make_tmap(&tw2s, w2, fp8, I, w2_rows, gemm_weight_box_rows(Orient::kSwap, Proj::kW2)));
    MOE_TRY(make_tmap(&txs, xperm, fp8, H, A, gemm_token_box_rows(Orient::kSwap)));
    MOE_TRY(make_tmap(&tis, inter, fp8, I, A, gemm_token_box_rows(Orient::kSwap)));
  }
  if (any_normal) {
    MOE_TRY(make_tmap(&tw13n, w13, fp8, H, w13_rows, gemm_weight_box_rows(Orient::kNormal, Proj::kW13)));
    MOE_TRY(make_tmap(&tw2n, w2, fp8, I, w2_rows, gemm_weight_box_rows(Orient::kNormal, Proj::kW2)));
    if (w2_pair2sm_supported(H, fp8)) MOE_TRY(make_tmap(&tw2p, w2, fp8, I, w2_rows, 128));
    MOE_TRY(make_tmap(&txn, xperm, fp8, H, A, gemm_token_box_rows(Orient::kNormal)));
    MOE_TRY(make_tmap(&tin, inter, fp8, I, A, gemm_token_box_rows(Orient::kNormal)));
  }

  record(dbg, 0, st);
  RouterArgs ra{static_cast<const __nv_bfloat16*>(hidden), static_cast<const __nv_bfloat16*>(router_w),
                router_bias, T, H, E, k,
                at<float>(ws, L.logits), at<float>(ws, L.xnorm), at<float>(ws, L.wnorm),
                at<float>(ws, L.amax_tok), at<int32_t>(ws, L.topk_ids), at<float>(ws, L.topk_w),
                at<unsigned char>(ws, L.cand), hdr, at<float>(ws, L.rsplit), invariant ? 1 : 0,
                at<float>(ws, L.partials)};
  AlignArgs aa{at<int32_t>(ws, L.topk_ids), T, E, k,
               at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.perm),
               at<int32_t>(ws, L.inv_perm), at<int4>(ws, L.chunks_swap), at<int4>(ws, L.chunks_normal),
               at<int4>(ws, L.chunks_pair),
               tau, gemm_swap_chunk(), fp8 ? at<float>(ws, L.amax_tok) : nullptr, hdr,
               at<int>(ws, L.gemm_flags), L.n_gemm_flags, at<int>(ws, L.slice_hist)};
  // Decode-sized calls: the top-k kernel's last CTA runs the align (the
  // "router" stage then covers the align too and the "align" stage is empty).
  bool fused_route = false;
  const int grid = device_sm_count() < kMaxSlots ? device_sm_count() : kMaxSlots;
  const unsigned long long timeout_ns = (dbg && dbg->wait_timeout_us > 0)
                                            ? static_cast<unsigned long long>(dbg->wait_timeout_us) * 1000ull
                                            : kWaitTimeoutNs;
  if (tc_router_eligible(T, H, E, invariant))
    MOE_TRY(route_tc(ra, grid, timeout_ns, st, &aa, &fused_route));
  else
    MOE_TRY(cuda_status(launch_router(ra, st, invariant ? nullptr : &aa, &fused_route)));
  record(dbg, 1, st);
  if (!fused_route) MOE_TRY(cuda_status(launch_align(aa, st)));
  record(dbg, 2, st);

  MOE_TRY(cuda_status(launch_gather(static_cast<const __nv_bfloat16*>(hidden), at<int32_t>(ws, L.perm),
                                    A, k, H, fp8, hdr, xperm, st)));
  record(dbg, 3, st);

  int* flags = at<int>(ws, L.gemm_flags);   // one kMaxSlots array per GEMM launch
  GemmArgs g13{};
  g13.katoms = H * (fp8 ? 1 : 2) / kAtomBytes;
  g13.w_rows_per_expert = 2 * I;
  g13.up_offset = I;
  g13.out = fp8 ? at<void>(ws, L.h32) : inter;
  g13.ld_out = I;
  g13.perm = at<int32_t>(ws, L.perm);
  g13.counts = at<int32_t>(ws, L.counts);
  g13.topk_w = at<float>(ws, L.topk_w);
  g13.num_assign = A;
  g13.wscale = w13_scale;
  g13.act_scale = hdr + kHdrScaleS1;
  g13.hdr = hdr;
  g13.partials = at<float>(ws, L.partials);
  g13.timeout_ns = timeout_ns;
  g13.inject_stall = dbg ? dbg->inject_stall : 0;
  g13.whole_units = invariant ? 1 : 0;
  float* amax_cta = at<float>(ws, L.amax_cta);
  // FP8: the last gate/up launch of the call requantises the whole
  // intermediate after a grid barrier (per-tensor s2 over every launch's amax)
  const int n_amax = (any_swap ? grid : 0) + (any_normal ? grid : 0);
  auto requant_args = [&](GemmArgs& g, bool last) {
    g.amax_all = amax_cta;
    g.amax_n = (fp8 && last) ? n_amax : 0;
    g.inter_q = inter;
    g.requant_n4 = static_cast<long long>(A) * I / 4;
  };
  GemmArgs g2 = g13;
  g2.katoms = I * (fp8 ? 1 : 2) / kAtomBytes;
  g2.w_rows_per_expert = H;
  g2.up_offset = 0;
  g2.out = at<void>(ws, L.ysc);
  g2.ld_out = H;
  g2.wscale = w2_scale;
  g2.act_scale = hdr + kHdrScaleS2;
  g2.amax_cta = nullptr;
  g2.amax_n = 0;
  g2.inject_stall = 0;
  // Decode batches in bf16 (T <= 32, every expert swap-AB): both GEMMs in one
  // persistent launch (ffn.cu); otherwise one launch per GEMM and orientation.
  const bool use_ffn = !fp8 && !invariant && any_swap && !any_normal && ffn_swap_supported(T, H, I) &&
                       fused_ffn_enabled() && !(dbg && dbg->force_orient == 3);
  if (use_ffn) {
    GemmArgs a = g13;
    a.chunks = at<int4>(ws, L.chunks_swap);
    a.nchunks = hdr + kHdrChunksSwap;
    a.mtiles = I / kTileM;
    a.amax_cta = nullptr;
    a.amax_n = 0;
    a.flags = flags + 0 * kMaxSlots;
    GemmArgs b = g2;
    b.chunks = at<int4>(ws, L.chunks_swap);
    b.nchunks = hdr + kHdrChunksSwap;
    b.mtiles = H / kTileM;
    b.flags = flags + 2 * kMaxSlots;
    b.partials = at<float>(ws, L.partials2);
    MOE_TRY(cuda_status(launch_ffn_swap(tw13s, txs, tw2s, tis, a, b, flags + kGemmLaunches * kMaxSlots, grid, st)));
    record(dbg, 4, st);
    record(dbg, 5, st);
  } else {
    if (any_swap) {
      GemmArgs g = g13;
      g.chunks = at<int4>(ws, L.chunks_swap);
      g.nchunks = hdr + kHdrChunksSwap;
      g.mtiles = I / kTileM;
      g.amax_cta = amax_cta;
      g.flags = flags + 0 * kMaxSlots;
      requant_args(g, !any_normal);
      MOE_TRY(cuda_status(launch_gemm(Orient::kSwap, Proj::kW13, fp8, tw13s, txs, g, grid, st)));
    }
    if (any_normal) {
      GemmArgs g = g13;
      g.chunks = at<int4>(ws, L.chunks_pair);
      g.nchunks = hdr + kHdrChunksPair;
      g.mtiles = I / gemm_weight_box_rows(Orient::kNormal, Proj::kW13);
      g.amax_cta = amax_cta + (any_swap ? grid : 0);
      g.flags = flags + 1 * kMaxSlots;
      requant_args(g, true);
      if (w13_pair2sm_supported(I, fp8)) {
        MOE_TRY(cuda_status(launch_w13_pair2sm(tw13n, txn, g, grid, st)));
      } else {
        MOE_TRY(cuda_status(launch_gemm(Orient::kNormal, Proj::kW13, fp8, tw13n, txn, g, grid, st)));
      }
    }
    record(dbg, 4, st);   // (the FP8 requantisation ran at the end of the gate/up GEMM)
    record(dbg, 5, st);
    if (any_swap) {
      GemmArgs g = g2;
      g.chunks = at<int4>(ws, L.chunks_swap);
      g.nchunks = hdr + kHdrChunksSwap;
      g.mtiles = H / kTileM;
      g.flags = flags + 2 * kMaxSlots;
      MOE_TRY(cuda_status(launch_gemm(Orient::kSwap, Proj::kW2, fp8, tw2s, tis, g, grid, st)));
    }
    if (any_normal) {
      GemmArgs g = g2;
      g.flags = flags + 3 * kMaxSlots;
      if (w2_pair2sm_supported(H, fp8)) {
        g.chunks = at<int4>(ws, L.chunks_pair);
        g.nchunks = hdr + kHdrChunksPair;
        MOE_TRY(cuda_status(launch_w2_pair2sm(tw2p, tin, g, grid, st)));
      } else {
        g.chunks = at<int4>(ws, gemm_w2_pair() ? L.chunks_pair : L.chunks_normal);
        g.nchunks = hdr + (gemm_w2_pair() ? kHdrChunksPair : kHdrChunksNormal);
        g.mtiles = H / gemm_weight_box_rows(Orient::kNormal, Proj::kW2);
        MOE_TRY(cuda_status(launch_gemm(Orient::kNormal, Proj::kW2, fp8, tw2n, tin, g, grid, st)));
      }
    }
  }
  record(dbg, 6, st);
  // combine: out[t] = sum_j ysc[t*k + j] in slot order (fp32), one rounding
  MOE_TRY(cuda_status(launch_combine(at<float>(ws, L.ysc), T, k, H, out, out_fp32, st)));
  record(dbg, 7, st);

  if (dbg) {
    auto cp = [&](void* dst, size_t off, size_t bytes) -> cudaError_t {
      return dst ? cudaMemcpyAsync(dst, static_cast<char*>(ws) + off, bytes, cudaMemcpyDeviceToDevice, st)
                 : cudaSuccess;
    };
    MOE_TRY(cuda_status(cp(dbg->topk_ids, L.topk_ids, static_cast<size_t>(A) * 4)));
    MOE_TRY(cuda_status(cp(dbg->topk_w, L.topk_w, static_cast<size_t>(A) * 4)));
    MOE_TRY(cuda_status(cp(dbg->counts, L.counts, static_cast<size_t>(E) * 4)));
    MOE_TRY(cuda_status(cp(dbg->offsets, L.offsets, static_cast<size_t>(E + 1) * 4)));
    MOE_TRY(cuda_status(cp(dbg->perm, L.perm, static_cast<size_t>(A) * 4)));
    MOE_TRY(cuda_status(cp(dbg->inv_perm, L.inv_perm, static_cast<size_t>(A) * 4)));
    MOE_TRY(cuda_status(cp(dbg->inter, L.inter, static_cast<size_t>(A) * I * (fp8 ? 1 : 2))));
    if (dbg->act_scales)
      MOE_TRY(cuda_status(cudaMemcpyAsync(dbg->act_scales, hdr + kHdrScaleS1, 8, cudaMemcpyDeviceToDevice, st)));
    if (dbg->hidden_q && fp8)
      MOE_TRY(cuda_status(launch_unpermute_rows(xperm, at<int32_t>(ws, L.inv_perm), T, k, H, dbg->hidden_q, st)));
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Launch cache.  A layer call enqueues about ten kernels; a caller that
// repeats a call with identical arguments (a decode loop) gets it replayed
// from an instantiated CUDA graph, one host launch instead of ten.  The first
// call with a key runs directly (and performs every one-time initialisation);
// the second records the same enqueue sequence on an internal stream that is
// only ever captured, instantiates the graph and launches it on the caller's
// stream; later calls launch the cached graph.  Calls made while the caller's
// stream is being captured, and calls with debug outputs, run directly.  A
// graph reads its buffers at replay time, so new contents at the same
// addresses are seen; any change of pointer or size is a different key.
// Only calls whose every pointer is device memory are cached (a graph would
// keep host addresses in its copy nodes past the lifetime of the caller's
// pinned buffers).  One cache per device; the capture and instantiation run
// outside the cache's lock, so other threads are not held up by them (a call
// that finds its key being captured by another thread runs directly).
struct CallKey {
  int kind;
  const void* p[9];
  long long n[7];
  bool operator==(const CallKey& o) const {
    if (kind != o.kind) return false;
    for (int i = 0; i < 9; ++i)
      if (p[i] != o.p[i]) return false;
    for (int i = 0; i < 7; ++i)
      if (n[i] != o.n[i]) return false;
    return true;
  }
};

enum CacheState { kEmpty = 0, kSeenOnce = 1, kReady = 2, kFailed = 3, kCapturing = 4 };

struct CacheEntry {
  CallKey key;
  int state;
  cudaGraphExec_t exec;
  unsigned long long used;
};

constexpr int kCacheEntries = 32;

struct DeviceCache {
  std::mutex mu;
  CacheEntry e[kCacheEntries];
  cudaStream_t capture_stream = nullptr;
  unsigned long long clock = 0;
};

struct CacheStats {
  std::mutex mu;
  unsigned long long replays = 0, captures = 0, failures = 0, direct = 0;
};

CacheStats& cache_stats() {
  static CacheStats s;
  return s;
}

void count(unsigned long long CacheStats::*field) {
  CacheStats& s = cache_stats();
  std::lock_guard<std::mutex> lock(s.mu);
  ++(s.*field);
}

template <class Enqueue>
moe_status_t run_direct(cudaStream_t st, Enqueue&& enqueue) {
  count(&CacheStats::direct);
  return enqueue(st);
}

template <class Enqueue>
moe_status_t run_cached(int dev, const CallKey& key, cudaStream_t st, Enqueue&& enqueue) {
  static DeviceCache caches[kMaxDevices];
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (dev < 0 || dev >= kMaxDevices || cudaStreamIsCapturing(st, &cs) != cudaSuccess ||
      cs != cudaStreamCaptureStatusNone)
    return run_direct(st, enqueue);
  DeviceCache& c = caches[dev];
  CacheEntry* e = nullptr;
  cudaStream_t cap = nullptr;
  {
    std::lock_guard<std::mutex> lock(c.mu);
    for (int i = 0; i < kCacheEntries; ++i)
      if (c.e[i].state != kEmpty && c.e[i].key == key) e = &c.e[i];
    if (e == nullptr) {   // first sighting: remember the key, run directly
      CacheEntry* v = nullptr;
      for (int i = 0; i < kCacheEntries && v == nullptr; ++i)
        if (c.e[i].state == kEmpty) v = &c.e[i];
      for (int i = 0; i < kCacheEntries && v == nullptr; ++i) v = &c.e[i];
      for (int i = 0; i < kCacheEntries; ++i)   // least recently used, never one being captured
        if (c.e[i].state != kCapturing && c.e[i].used < v->used) v = &c.e[i];
      if (v->state == kCapturing) return run_direct(st, enqueue);
      if (v->state == kReady) cudaGraphExecDestroy(v->exec);
      *v = CacheEntry{key, kSeenOnce, nullptr, ++c.clock};
      return run_direct(st, enqueue);
    }
    e->used = ++c.clock;
    if (e->state == kReady) {
      const cudaError_t err = cudaGraphLaunch(e->exec, st);
      if (err == cudaSuccess) count(&CacheStats::replays);
      return cuda_status(err);
    }
    if (e->state != kSeenOnce) return run_direct(st, enqueue);   // failed, or another thread captures
    if (c.capture_stream == nullptr &&
        cudaStreamCreateWithFlags(&c.capture_stream, cudaStreamNonBlocking) != cudaSuccess) {
      c.capture_stream = nullptr;
      e->state = kFailed;
      count(&CacheStats::failures);
      return run_direct(st, enqueue);
    }
    e->state = kCapturing;
    cap = c.capture_stream;
  }
  // second sighting: record outside the lock (only this thread uses `cap`
  // while the entry is marked as capturing, and an entry being captured is
  // never evicted)
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  bool ok = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
  if (ok) {
    const moe_status_t rc = enqueue(cap);
    const cudaError_t end = cudaStreamEndCapture(cap, &graph);
    ok = rc == MOE_OK && end == cudaSuccess && graph != nullptr;
    if (ok) ok = cudaGraphInstantiate(&exec, graph, 0ULL) == cudaSuccess;
    if (graph != nullptr) cudaGraphDestroy(graph);
  }
  cudaGetLastError();   // a failed capture leaves no sticky error
  {
    std::lock_guard<std::mutex> lock(c.mu);
    e->state = ok ? kReady : kFailed;
    e->exec = ok ? exec : nullptr;
  }
  count(ok ? &CacheStats::captures : &CacheStats::failures);
  if (!ok) return run_direct(st, enqueue);
  const cudaError_t err = cudaGraphLaunch(exec, st);
  if (err == cudaSuccess) count(&CacheStats::replays);
  return cuda_status(err);
}

int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(int T, int H, int E, int I, int top_k, int dtype) {
  if (check_shape(T, H, E, I, top_k, dtype) != MOE_OK) return 0;
  return make_layout(T, H, E, I, top_k, dtype == MOE_DTYPE_FP8_E4M3).total;
}

moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < static_cast<size_t>(kHeaderBytes)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward(const void* hidden, const void* router_w, const float* router_bias,
                         const void* w13, const void* w2, const float* w13_scale,
                         const float* w2_scale, int T, int H, int E, int I, int top_k, int dtype,
                         void* out, void* workspace, size_t workspace_bytes, moe_debug_out_t* dbg,
                         void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto enqueue = [&](cudaStream_t s) {
    return forward_impl(hidden, router_w, router_bias, w13, w2, w13_scale, w2_scale, T, H, E, I,
                        top_k, dtype, out, workspace, workspace_bytes, dbg, s);
  };
  if (dbg != nullptr || check_shape(T, H, E, I, top_k, dtype) != MOE_OK) return enqueue(st);
  const CallKey key{0, {hidden, router_w, router_bias, w13, w2, w13_scale, w2_scale, out, workspace},
                    {T, H, E, I, top_k, dtype, static_cast<long long>(workspace_bytes)}};
  return run_cached(current_device(), key, st, enqueue);
}

moe_status_t moe_forward_batch_invariant(const void* hidden, const void* router_w,
                                         const float* router_bias, const void* w13, const void* w2,
                                         int T, int H, int E, int I, int top_k, void* out,
                                         void* workspace, size_t workspace_bytes,
                                         moe_debug_out_t* dbg, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto enqueue = [&](cudaStream_t s) {
    return forward_impl(hidden, router_w, router_bias, w13, w2, nullptr, nullptr, T, H, E, I,
                        top_k, MOE_DTYPE_BF16, out, workspace, workspace_bytes, dbg, s, true);
  };
  if (dbg != nullptr || check_shape(T, H, E, I, top_k, MOE_DTYPE_BF16) != MOE_OK) return enqueue(st);
  const CallKey key{1, {hidden, router_w, router_bias, w13, w2, nullptr, nullptr, out, workspace},
                    {T, H, E, I, top_k, MOE_DTYPE_BF16, static_cast<long long>(workspace_bytes)}};
  return run_cached(current_device(), key, st, enqueue);
}

moe_status_t moe_forward_hostio(const void* hidden_host, const void* router_w,
                                const float* router_bias, const void* w13, const void* w2,
                                const float* w13_scale, const float* w2_scale, int T, int H, int E,
                                int I, int top_k, int dtype, void* out_host, void* workspace,
                                size_t workspace_bytes, void* stream) {
  MOE_TRY(check_shape(T, H, E, I, top_k, dtype));
  if (!hidden_host || !out_host || !workspace) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(T, H, E, I, top_k, dtype == MOE_DTYPE_FP8_E4M3);
  if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* din = at<void>(workspace, L.staging_in);
  void* dout = at<void>(workspace, L.staging_out);
  const size_t bytes = static_cast<size_t>(T) * H * 2;
  // Enqueued directly, never replayed from a cached graph: a graph would hold
  // the host addresses in its copy nodes, and a later buffer at the same
  // address need not be pinned.
  MOE_TRY(cuda_status(cudaMemcpyAsync(din, hidden_host, bytes, cudaMemcpyHostToDevice, st)));
  MOE_TRY(forward_impl(din, router_w, router_bias, w13, w2, w13_scale, w2_scale, T, H, E, I, top_k,
                       dtype, dout, workspace, workspace_bytes, nullptr, st));
  return cuda_status(cudaMemcpyAsync(out_host, dout, bytes, cudaMemcpyDeviceToHost, st));
}

moe_status_t moe_forward_partial(const void* hidden, const void* router_w, const float* router_bias,
                                 const void* w13_shard, const void* w2_shard, const float* w13_scale,
                                 const float* w2_scale, int T, int H, int E, int I_shard, int top_k,
                                 int dtype, float* out_partial, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  return forward_impl(hidden, router_w, router_bias, w13_shard, w2_shard, w13_scale, w2_scale, T, H, E,
                      I_shard, top_k, dtype, out_partial, workspace, workspace_bytes, nullptr,
                      static_cast<cudaStream_t>(stream), false, true);
}

moe_status_t moe_sum_partials(const float* partials, int G, int T, int H, void* out, void* stream) {
  if (!partials || !out) return MOE_ERR_INVALID_ARG;
  if (G < 1 || T < 1 || H < 128 || H > 8192 || H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(partials) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  return cuda_status(launch_sum_partials(partials, G, static_cast<long long>(T) * H,
                                         static_cast<__nv_bfloat16*>(out), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_inv_rope_fp8_quant(const void* x, const int32_t* positions, const float* cos_tab,
                                    const float* sin_tab, int T, int n_heads, int head_dim, int max_pos,
                                    uint8_t* codes, float* scales, void* stream) {
  if (!x || !positions || !cos_tab || !sin_tab || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (T < 1 || n_heads < 1 || max_pos < 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (head_dim != 16 && head_dim != 32 && head_dim != 64 && head_dim != 128 && head_dim != 256 &&
      head_dim != 512)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * n_heads * head_dim >= (1LL << 40)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(cos_tab) || !aligned16(sin_tab) || !aligned16(codes) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u))
    return MOE_ERR_MISALIGNED;
  return cuda_status(launch_inv_rope_fp8(x, positions, cos_tab, sin_tab, T, n_heads, head_dim, max_pos, codes,
                                         scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route(const void* hidden, const void* router_w, const float* router_bias, int T,
                       int H, int E, int top_k, int32_t* topk_ids, float* topk_w, void* workspace,
                       size_t workspace_bytes, void* stream) {
  MOE_TRY(check_shape(T, H, E, 128, top_k, MOE_DTYPE_BF16));
  if (!hidden || !router_w || !topk_ids || !topk_w || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(router_w) || !aligned16(workspace)) return MOE_ERR_MISALIGNED;
  const Layout L = make_layout(T, H, E, 128, top_k, false);
  if (workspace_bytes < L.rsplit + router_split_floats(T, E) * 4) return MOE_ERR_WORKSPACE_TOO_SMALL;
  RouterArgs ra{static_cast<const __nv_bfloat16*>(hidden), static_cast<const __nv_bfloat16*>(router_w),
                router_bias, T, H, E, top_k,
                at<float>(workspace, L.logits), at<float>(workspace, L.xnorm),
                at<float>(workspace, L.wnorm), at<float>(workspace, L.amax_tok), topk_ids, topk_w,
                at<unsigned char>(workspace, L.cand), at<uint32_t>(workspace, L.header),
                at<float>(workspace, L.rsplit), 0, at<float>(workspace, L.partials)};
  if (tc_router_eligible(T, H, E, false)) {
    const int grid = device_sm_count() < kMaxSlots ? device_sm_count() : kMaxSlots;
    return route_tc(ra, grid, kWaitTimeoutNs, static_cast<cudaStream_t>(stream));
  }
  return cuda_status(launch_router(ra, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_align(const int32_t* topk_ids, int T, int E, int top_k, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (E < 1 || E > kMaxExperts || top_k < 1 || top_k > kMaxTopK || T < 1 ||
      static_cast<long long>(T) * top_k > (1LL << 24))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!topk_ids || !counts || !offsets || !perm || !inv_perm || !workspace) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(T, 128, E, 128, top_k, false);
  if (workspace_bytes < L.gemm_flags + static_cast<size_t>(L.n_gemm_flags) * 4) return MOE_ERR_WORKSPACE_TOO_SMALL;
  AlignArgs aa{topk_ids, T, E, top_k, counts, offsets, perm, inv_perm,
               at<int4>(workspace, L.chunks_swap), at<int4>(workspace, L.chunks_normal),
               at<int4>(workspace, L.chunks_pair),
               swap_threshold(), gemm_swap_chunk(), nullptr, at<uint32_t>(workspace, L.header),
               at<int>(workspace, L.gemm_flags), L.n_gemm_flags,
               at<int>(workspace, L.slice_hist)};
  return cuda_status(launch_align(aa, static_cast<cudaStream_t>(stream)));
}

void moe_cache_stats(unsigned long long* out4) {
  if (!out4) return;
  CacheStats& s = cache_stats();
  std::lock_guard<std::mutex> lock(s.mu);
  out4[0] = s.replays;
  out4[1] = s.captures;
  out4[2] = s.failures;
  out4[3] = s.direct;
}

moe_status_t moe_get_status(void* workspace, void* stream, uint32_t* info_out) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(h), st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (info_out) *info_out = h[1];
  return static_cast<moe_status_t>(h[0]);
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "expert id out of range";
    case MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case MOE_ERR_EXCEEDS_STATIC_SCRATCH: return "shape exceeds the fixed static scratch";
  }
  return "unknown status";
}

}  // extern "C"
