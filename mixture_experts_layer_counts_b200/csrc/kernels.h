// Host-side launch wrappers of the library's kernels (internal interface
// between the C ABI in api.cu and the kernel translation units).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace moe {

// Raises a kernel's dynamic shared-memory limit to at least `bytes`, once per
// (kernel, device); later calls with the same or a smaller size do nothing.
cudaError_t set_smem_limit_once(const void* kernel, int bytes);

// Multiprocessor count of the current device (cached per device).
int current_sm_count();

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel on the stream is still running, and must execute
// griddepcontrol.wait (pdl_wait) before it reads anything that kernel wrote.
template <typename... KParams, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KParams...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KParams>(args)...);
}

#ifdef __CUDACC__
// Device side of a programmatic launch: wait for the previous kernel's
// results, then let the next kernel on the stream be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

struct RouterArgs {
  const __nv_bfloat16* hidden;
  const __nv_bfloat16* router_w;
  const float* bias;
  int T, H, E, k;
  float* logits;
  float* xnorm;
  float* wnorm;
  float* amax_tok;
  int32_t* topk_ids;
  float* topk_w;
  unsigned char* cand;
  uint32_t* hdr;
  float* rsplit;          // router_split_floats(T, E) floats, or NULL (no split-K)
  int invariant;          // 1: one logits kernel and summation order for every T (no split-K)
  float* partials;        // GEMM partial tiles for the tensor-core logits (NULL: whole units)
};
struct AlignArgs;
// fuse_align non-NULL and MOE_FUSE_ALIGN=1: a decode-sized call lets the
// top-k kernel's last CTA run the align (then *fused is set and the align
// must not be launched again); by default the align is its own launch.
cudaError_t launch_router(const RouterArgs& a, cudaStream_t st, const AlignArgs* fuse_align = nullptr,
                          bool* fused = nullptr);
// The top-k of logits from the tensor cores (logits, norms and amax already
// written), with the relative error bound `gamma` of the logits (times
// ||x|| ||w||) and `ulast` of their last roundings: one warp per token, every
// candidate within twice the bound of the k-th re-evaluated in mixed
// precision (in fp64 where that leaves the order open).  With
// `aa` non-NULL a decode-sized call's last CTA also runs the align (*fused set).
cudaError_t launch_router_topk_tc(const RouterArgs& a, float gamma, float ulast, cudaStream_t st,
                                  const AlignArgs* aa = nullptr, bool* fused = nullptr);

struct AlignArgs {
  const int32_t* topk_ids;
  int T, E, k;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  int4* chunks_swap;
  int4* chunks_normal;
  int4* chunks_pair;      // normal orientation, 256-token chunks (gate/up GEMM)
  int swap_max_count;     // experts with count <= this run swap-AB
  int swap_chunk;         // tokens per swap-AB chunk (the swap kernels' largest N)
  const float* amax_tok;  // FP8: per-token amax|x| (NULL on bf16)
  uint32_t* hdr;
  int* gemm_flags;        // split-tile flags of the GEMM launches, zeroed here (may be NULL)
  int n_gemm_flags;
  int* slice_hist;        // kAlignMaxSlices * E ints for large T*k (NULL: one CTA)
};
cudaError_t launch_align(const AlignArgs& a, cudaStream_t st);

// x_perm[p, :] = hidden[perm[p] / k, :]   (bf16 copy, or E4M3 of x / s1 on FP8)
cudaError_t launch_gather(const __nv_bfloat16* hidden, const int32_t* perm, int A, int k, int H,
                          bool fp8, const uint32_t* hdr, void* xperm, cudaStream_t st);

// Debug output: dst[t, :] = src[inv_perm[t * k], :] for rows of row_bytes (a multiple of 16)
cudaError_t launch_unpermute_rows(const void* src, const int32_t* inv_perm, int T, int k, int row_bytes,
                                  void* dst, cudaStream_t st);


// Inverse RoPE + per-head E4M3 quantisation (rope.cu); D in {16, 32, 64, 128, 256, 512}
cudaError_t launch_inv_rope_fp8(const void* x, const int32_t* pos, const float* cos_tab, const float* sin_tab,
                                int T, int nH, int D, int max_pos, uint8_t* codes, float* scales,
                                cudaStream_t st);

// out[t, :] = bf16( sum_{j<k} ysc[t*k + j, :] ), j ascending (fp32 sum), or the fp32 sum
cudaError_t launch_combine(const float* ysc, int T, int k, int H, void* out, bool out_f32, cudaStream_t st);

// out[t, :] = bf16( sum_{g < G} parts[g, t, :] ), g ascending (fp32 sum)
cudaError_t launch_sum_partials(const float* parts, int G, long long n, __nv_bfloat16* out, cudaStream_t st);

struct GemmArgs {
  const int4* chunks;          // {expert, first row in perm order, rows, index inside expert}
  const uint32_t* nchunks;     // header word holding the chunk count
  const int32_t* counts;       // [E] assignments per expert (normal orientation: chunks of e)
  int mtiles;                  // weight tiles per chunk
  int katoms;                  // K / 128 bytes
  int w_rows_per_expert;       // rows of one expert in the 2-D weight view
  int up_offset;               // w13: row offset of the up half (= I)
  void* out;                   // w13: inter (bf16) or h32 (fp32, FP8); w2: ysc (fp32)
  int ld_out;
  const int32_t* perm;
  const float* topk_w;
  int num_assign;              // T * top_k (bounds of perm values)
  const float* wscale;         // FP8 per-expert weight scale
  const uint32_t* act_scale;   // FP8: header word with s1 (w13) or s2 (w2)
  float* amax_cta;             // FP8 w13: per-CTA amax|h| (this launch's slots)
  const float* amax_all;       // FP8 w13, last launch of the call: every launch's per-CTA amax ...
  int amax_n;                  // ... (amax_n slots); > 0 makes this launch requantise the whole
  void* inter_q;               // intermediate into inter_q (E4M3) after a grid barrier
  long long requant_n4;        // A * I / 4
  uint32_t* hdr;
  float* partials;             // kMaxSlots fp32 partial tiles (split units)
  int* flags;                  // kMaxSlots flags, zero at launch
  int flags_self_reset;        // 1: the CTA that consumes a split unit's flags zeroes them again
                               // (flags that no align kernel clears, e.g. the router's)
  unsigned long long timeout_ns;   // limit of every bounded wait in the kernel
  int inject_stall;            // failure-path test: CTA 0 leaves one stage unfilled
  // Router logits mode of the swap-AB down-projection kernel (dense_T > 0):
  // weight rows = router rows (n_cols experts), token chunks = dense tiles of
  // the hidden rows (no schedule, no perm), out = logits [dense_T, n_cols] fp32
  // with col_bias added; the epilogue warps first write the norms the
  // router's certification needs (||x_t||, amax|x_t|, ||w_e||).
  int dense_T;
  int dense_chunk;             // tokens per dense chunk (the swap-AB kernel's largest N)
  int n_cols;
  const float* col_bias;
  const void* norm_x;          // hidden [dense_T, norm_H] bf16
  const void* norm_w;          // router_w [n_cols, norm_H] bf16
  float* xnorm;
  float* wnorm;
  float* amax_tok;
  int norm_H;
  int whole_units;             // 1: whole units dealt round-robin (no K splits) and, for
                               // swap-AB, MMA N fixed at the largest chunk: every output
                               // element then sees the same operations whatever the batch
};

// Fused expert FFN of decode batches (ffn.cu): gate/up and down GEMMs, swap-AB,
// bf16, one persistent launch; chunks of at most ffn_swap_chunk() tokens.
bool ffn_swap_supported(int T, int H, int I);
int ffn_swap_chunk();
cudaError_t launch_ffn_swap(const CUtensorMap& tw13, const CUtensorMap& tx, const CUtensorMap& tw2,
                            const CUtensorMap& th, const GemmArgs& g13, const GemmArgs& g2, int* dep, int grid,
                            cudaStream_t st);

enum class Orient { kSwap, kNormal };
enum class Proj { kW13, kW2 };
cudaError_t launch_gemm(Orient o, Proj p, bool fp8, const CUtensorMap& tm_w,
                        const CUtensorMap& tm_x, const GemmArgs& a, int grid, cudaStream_t st);
bool gemm_w2_pair();
// Normal-orientation GEMMs on CTA pairs (gemm2sm.cu), bf16, 256-token chunks:
// gate/up with I a multiple of 256, down with H a multiple of 512.  Both take
// 128-row boxes in their tensor maps.  MOE_W13_2SM=0 / MOE_W2_2SM=0 keep the
// one-CTA kernels (for measurements).
bool w13_pair2sm_supported(int I, bool fp8);
bool w2_pair2sm_supported(int H, bool fp8);
cudaError_t launch_w13_pair2sm(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int max_ctas,
                               cudaStream_t st);
cudaError_t launch_w2_pair2sm(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int max_ctas,
                              cudaStream_t st);                 // normal down GEMM on 256-token chunks (two M tiles)
int gemm_token_box_rows(Orient o);   // rows per TMA box of the token operand
int gemm_swap_chunk();               // largest token chunk of the swap-AB kernels
int gemm_weight_box_rows(Orient o, Proj p);

}  // namespace moe
