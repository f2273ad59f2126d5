/*
 * moe.h -- C ABI of the B200 (sm_100a) fused Mixture-of-Experts layer.
 *
 * What it computes.  Fused MoE is one batched GPU operation covering token
 * routing, the movement of token data and the experts' arithmetic ("AWS
 * describes a fused MoE optimization for the NVIDIA Hopper architecture",
 * body), with scaling, matrix products and the aggregation of expert outputs
 * done in one pass ("AWS details MoE kernel fixes for SageMaker, upstreams
 * them to vLLM", paragraph on the Triton backend).  For each token t:
 *   logits[e] = hidden[t] . router_w[e] (+ router_bias[e])
 *   p         = fp32 softmax over the E logits
 *   ids       = the top_k experts by logit, descending, exact ties -> lower id
 *   w[j]      = p[ids[j]] / sum_j' p[ids[j']]
 *   for each slot j, expert e = ids[j]:
 *       g = W1[e] x, u = W3[e] x   (W1 = rows [0,I) of w13[e], W3 = rows [I,2I))
 *       h = SiLU(g) * u            (rounded to bf16, or E4M3 on the FP8 path)
 *       y = W2[e] h
 *   out[t] = bf16( sum_j w[j] * y_j )   (fp32 sum in slot order j = 0..top_k-1)
 * The Hopper "Swap-AB" operand swap the pages describe ("AWS Unveils MoE
 * Kernel Optimizations...", Swap-AB section) becomes a per-expert choice of
 * tcgen05 orientation inside the library: experts with few tokens put the
 * weight rows in the MMA's M slot and the tokens in N; experts with many
 * tokens use the normal orientation.
 *
 * Conventions for every entry point:
 *  - Pointers named *_host are host memory (pinned for asynchrony); every
 *    other pointer is device memory owned by the caller.  The library never
 *    allocates or frees memory on these calls; scratch space comes from the
 *    caller's workspace (moe_workspace_size).
 *  - All device pointers must be 16-byte aligned.  Matrices are row-major and
 *    densely packed.  bf16 = IEEE bfloat16 bit patterns (uint16); E4M3 = OCP
 *    FP8 E4M3FN codes (uint8).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream: they enqueue kernels
 *    and return.  Argument errors are returned synchronously and nothing is
 *    enqueued.  Errors found on the device (a wait that timed out, an expert
 *    id out of range) are recorded in the workspace's status word and read
 *    with moe_get_status.
 *  - Repeated calls of moe_forward / moe_forward_batch_invariant (without
 *    debug outputs) with identical arguments are replayed from a CUDA graph
 *    the library records on the second such call (on an internal stream;
 *    nothing runs during the recording) and keeps for up to 32 argument sets
 *    per device.  Buffers are read at replay time.  Calls on a stream that is
 *    being captured always enqueue their kernels directly.  A caller that
 *    passes the same out and workspace buffers on every call benefits; a new
 *    address is a new argument set.  moe_forward_hostio is never replayed
 *    from a graph (its host buffers may not outlive the call).
 *  - Shapes are runtime values; nothing is specialised per T (the pages'
 *    lesson about per-token-count JIT recompiles, "AWS details MoE kernel
 *    fixes...", third fix).  Results are deterministic: identical inputs give
 *    bit-identical outputs.
 *  - Limits: 1 <= T, T*top_k <= 2^24; 1 <= E <= 1024; 1 <= top_k <= min(E, 32);
 *    H and I multiples of 128 with 128 <= H <= 8192, 128 <= I <= 16384.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_DTYPE_BF16 = 0,     /* bf16 weights and activations, fp32 accumulate, bf16 out */
  MOE_DTYPE_FP8_E4M3 = 1  /* E4M3 weights (one fp32 scale per expert matrix), dynamic
                             per-tensor E4M3 activations and intermediate, bf16 out */
} moe_dtype_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* NULL pointer, bad dtype, top_k out of range */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* a size outside the limits above */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,
  MOE_ERR_CUDA = 4,               /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5,     /* a bounded device-side wait expired */
  MOE_ERR_DEVICE_BOUNDS = 6,      /* an expert id outside [0, E) reached moe_align */
  MOE_ERR_MISALIGNED = 7,         /* a pointer is not 16-byte aligned */
  MOE_ERR_EXCEEDS_STATIC_SCRATCH = 8  /* moe_route_static: T and E need more than its
                                         fixed 8 MiB scratch */
} moe_status_t;

/* Optional outputs of moe_forward for checking and profiling; every field may
 * be NULL.  Device pointers unless noted. */
typedef struct {
  int32_t *topk_ids;   /* [T, top_k] expert ids, slot order */
  float *topk_w;       /* [T, top_k] renormalised fp32 weights */
  int32_t *counts;     /* [E] assignments per expert */
  int32_t *offsets;    /* [E+1] exclusive prefix sum of counts */
  int32_t *perm;       /* [T*top_k] flat index t*top_k+j, grouped by expert, ascending inside */
  int32_t *inv_perm;   /* [T*top_k] inverse of perm */
  void *inter;         /* [T*top_k, I] intermediate h in perm order (bf16 or E4M3 codes) */
  float *act_scales;   /* [2] FP8 path: s1 (activations), s2 (intermediate) */
  void **stage_events; /* host array of 8 cudaEvent_t recorded on `stream` at the stage
                          boundaries: start, router, align, gather, w13, requant, w2, combine */
  int force_orient;    /* 0 = per-expert choice, 1 = swap-AB for all experts,
                          2 = normal orientation for all experts, 3 = swap-AB for all
                          experts with one launch per GEMM (no fused decode FFN)
                          (testing) */
  int wait_timeout_us; /* limit of each bounded device-side wait (0 = 2 s) */
  int inject_stall;    /* failure-path test: 1 makes the first gate/up GEMM CTA leave one
                          pipeline stage unfilled, so a bounded wait expires and the call
                          records MOE_ERR_DEVICE_TIMEOUT (the output is then undefined) */
  uint8_t *hidden_q;   /* [T, H] FP8 path: the E4M3 codes of hidden / s1 that the gate/up
                          GEMM consumed, in token order */
} moe_debug_out_t;

/* Bytes of workspace moe_forward needs for this shape (0 if the shape is
 * outside the limits).  The workspace holds routing results, the grouped
 * activations, the intermediate and the per-slot fp32 down-projection rows. */
size_t moe_workspace_size(int T, int H, int E, int I, int top_k, int dtype);

/* Zero the workspace's header (its first 1024 bytes: the status words and the
 * counters and flags that every call leaves at zero again).  Call once on a
 * fresh workspace before its first use, and again after a call that failed. */
moe_status_t moe_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* The whole layer.
 *   hidden     [T, H] bf16                 router_w   [E, H] bf16
 *   router_bias[E] fp32 or NULL: added to the logits before the softmax
 *   w13        [E, 2I, H] bf16 or E4M3     w2         [E, H, I] bf16 or E4M3
 *   w13_scale, w2_scale [E] fp32 (FP8 only, else NULL): weight = code * scale
 *   out        [T, H] bf16, written fully
 *   workspace  >= moe_workspace_size(...) bytes, initialised by moe_workspace_init
 *   dbg        NULL in production
 * Errors: MOE_ERR_INVALID_ARG / UNSUPPORTED_SHAPE / MISALIGNED /
 * WORKSPACE_TOO_SMALL before any launch; MOE_ERR_CUDA if a launch fails. */
moe_status_t moe_forward(const void *hidden, const void *router_w, const float *router_bias,
                         const void *w13, const void *w2, const float *w13_scale,
                         const float *w2_scale, int T, int H, int E, int I, int top_k, int dtype,
                         void *out, void *workspace, size_t workspace_bytes,
                         moe_debug_out_t *dbg, void *stream);

/* Batch-invariant form of moe_forward (bf16 only): the output row of a
 * token is bit-identical whatever other tokens share the call and whatever
 * its position in the batch.  (The pages' second theme is bit-exact
 * inference across processes for RL, "Fused MoE on Hopper, bit-exact vLLM
 * across processes, and linear attention on TPUs", TL;DR and key points;
 * this mode gives the layer that property with respect to batching.)  Every
 * element is produced by the same sequence of operations for any T: one
 * logits kernel with a fixed summation order (no split over H), exact
 * routing, the swap-AB orientation for every expert with the MMA's token
 * dimension fixed at 64, whole tiles per CTA (no split of the reduction
 * dimension across CTAs), and the slot-ordered combine.  Same arguments,
 * workspace (bf16) and errors as moe_forward, without the dtype and FP8
 * scale arguments: per-tensor FP8 scales depend on the whole batch, so this
 * mode is bf16 only.  Slower than moe_forward for large T (no normal
 * orientation, no split of the reduction across CTAs). */
moe_status_t moe_forward_batch_invariant(const void *hidden, const void *router_w,
                                         const float *router_bias, const void *w13, const void *w2,
                                         int T, int H, int E, int I, int top_k, void *out,
                                         void *workspace, size_t workspace_bytes,
                                         moe_debug_out_t *dbg, void *stream);

/* moe_forward with host-side activations: copies hidden_host [T, H] bf16
 * (pinned host memory) into the workspace, runs the layer, and copies the
 * result into out_host [T, H] bf16 (pinned host memory), all enqueued on
 * `stream`.  The caller synchronises the stream before reading out_host.
 * Weights stay device pointers. */
moe_status_t moe_forward_hostio(const void *hidden_host, const void *router_w,
                                const float *router_bias, const void *w13, const void *w2,
                                const float *w13_scale, const float *w2_scale, int T, int H,
                                int E, int I, int top_k, int dtype, void *out_host,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Tensor parallelism over the intermediate dimension I.  The pages' serving
 * figures come from 8-way tensor-parallel deployments ("AWS details MoE kernel
 * fixes for SageMaker, upstreams them to vLLM", The facts); for this layer the
 * split that stays balanced under skewed routing is over I: rank g of G holds
 * rows [g I/G, (g+1) I/G) of every expert's gate and up projections and the
 * matching columns of its down projection, so every rank streams 1/G of
 * every active expert.  h = SiLU(g) * u of an intermediate column depends
 * only on that column's gate and up rows, so the bf16 intermediate is the
 * same as without the split; the output is the sum over ranks of
 *   partial_g[t] = sum_j w[t, j] * W2[e][:, slice g] h[slice g].
 *
 * moe_forward_partial: the layer on one rank's slice.  Same arguments and
 * errors as moe_forward, with
 *   w13_shard [E, 2 * I_shard, H]: rows [0, I_shard) this rank's gate rows,
 *             rows [I_shard, 2 * I_shard) its up rows (bf16 or E4M3)
 *   w2_shard  [E, H, I_shard]: the matching columns of w2
 *   out_partial [T, H] fp32 (device): the unrounded slot-ordered sum above
 *   workspace >= moe_workspace_size(T, H, E, I_shard, top_k, dtype)
 * Routing is computed on every rank from the replicated hidden and router
 * weights; it is deterministic, so every rank routes identically.  FP8: the
 * activation scale s1 is the same on every rank; the intermediate scale s2
 * is taken over this rank's slice of h (a scale per shard, not per tensor).
 *
 * moe_sum_partials: out[t, :] = bf16( sum_{g=0..G-1} partials[g, t, :] ),
 * the fp32 partials added in rank order from g = 0 and rounded once, so
 * every rank that holds the gathered partials [G, T, H] (fp32, device)
 * computes the same bits.  out [T, H] bf16 (device).  The exchange of the
 * partials between ranks (an all-gather into local memory) is the caller's
 * collective. */
moe_status_t moe_forward_partial(const void *hidden, const void *router_w, const float *router_bias,
                                 const void *w13_shard, const void *w2_shard, const float *w13_scale,
                                 const float *w2_scale, int T, int H, int E, int I_shard, int top_k,
                                 int dtype, float *out_partial, void *workspace, size_t workspace_bytes,
                                 void *stream);

moe_status_t moe_sum_partials(const float *partials, int G, int T, int H, void *out, void *stream);

/* Fused inverse rotary position embedding + per-head FP8 quantisation, the
 * kernel the pages name as the third MoE serving fix (a fused RoPE + FP8
 * quantisation kernel, per head, whose token count must stay a runtime value:
 * "AWS details MoE kernel fixes for SageMaker, upstreams them to vLLM", third
 * fix; "AWS Unveils MoE Kernel Optimizations...", "Eliminating Triton JIT
 * Recompilation").  Nothing here is specialised per T.
 *   x         [T, n_heads, head_dim] bf16 (device), head vectors that carry RoPE
 *   positions [T] int32 (device), the table row of each token
 *   cos_tab, sin_tab [max_pos, head_dim / 2] fp32 (device), the rotary table
 *   codes     [T, n_heads, head_dim] E4M3 (device), scales [T, n_heads] fp32 (device)
 * For each token and head, element i < D/2 pairs with element i + D/2 and the
 * pair turns by minus its angle (c = cos_tab[pos, i], s = sin_tab[pos, i]):
 *   y[i] = x[i] c + x[i + D/2] s,   y[i + D/2] = x[i + D/2] c - x[i] s
 * in fp32 with every product and every sum rounded (no fused multiply-add);
 * then scale = fp32(max |y|) / 448 (1 when the head is all zeros) and codes =
 * E4M3(fp32(y / scale)), round-to-nearest-even, saturating to +-448.  A
 * position outside [0, max_pos) gives that token's heads codes 0 and scale 0.
 * head_dim in {16, 32, 64, 128, 256, 512}; x, the tables and codes 16-byte
 * aligned; positions and scales 4-byte aligned.  Errors: INVALID_ARG (NULL),
 * UNSUPPORTED_SHAPE, MISALIGNED before any launch; MOE_ERR_CUDA if the
 * launch fails.  Asynchronous on `stream`; needs no workspace. */
moe_status_t moe_inv_rope_fp8_quant(const void *x, const int32_t *positions, const float *cos_tab,
                                    const float *sin_tab, int T, int n_heads, int head_dim, int max_pos,
                                    uint8_t *codes, float *scales, void *stream);

/* Router only: topk_ids [T, top_k] int32 and topk_w [T, top_k] fp32 (device),
 * same definition as in moe_forward.  Uses the workspace of moe_forward's
 * shape (moe_workspace_size with the same T, H, E, top_k; any I >= 128). */
moe_status_t moe_route(const void *hidden, const void *router_w, const float *router_bias,
                       int T, int H, int E, int top_k, int32_t *topk_ids, float *topk_w,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Align only: group the T*top_k assignments in topk_ids by expert.
 * counts [E], offsets [E+1], perm and inv_perm [T*top_k] (device, int32),
 * bit-exact stable counting sort.  Ids outside [0, E) set
 * MOE_ERR_DEVICE_BOUNDS in the status word and are skipped. */
moe_status_t moe_align(const int32_t *topk_ids, int T, int E, int top_k, int32_t *counts,
                       int32_t *offsets, int32_t *perm, int32_t *inv_perm, void *workspace,
                       size_t workspace_bytes, void *stream);

/* Router for callers that cannot allocate device memory.  (No counterpart in
 * the pages: it is an interface of this library, not part of the method.)
 * Same computation and outputs as moe_route, but with no workspace argument:
 * its scratch is one 8 MiB array inside the library, fixed at build time.
 * Meant for code that receives its input and output buffers from a host
 * program but has no allocator of its own (a plug-in inside a runtime that
 * owns all device memory, or a hot loop that must not allocate).
 *   - Allocates nothing: no cudaMalloc / cudaFree, no library allocator.
 *   - The array exists on every GPU that loads this library, until exit.
 *   - Capacity: 20 * T * E + 4 * (2T + E) bytes plus alignment must fit in
 *     8 MiB (about T * E <= 400,000, e.g. T = 2048 with E = 128); larger
 *     shapes return MOE_ERR_EXCEEDS_STATIC_SCRATCH before anything runs.
 *   - The first call on a device looks up the array's device address; make
 *     that first call outside any stream capture.
 *   - All calls share the array: calls that may overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the caller.
 *   - Device-side status words live in the array too and are cleared at the
 *     start of every call; moe_get_status does not apply. */
moe_status_t moe_route_static(const void *hidden, const void *router_w, const float *router_bias,
                              int T, int H, int E, int top_k, int32_t *topk_ids, float *topk_w,
                              void *stream);

/* Counters of the launch cache since the library was loaded, for tests and
 * diagnostics: out4[0] graph launches (replays), out4[1] graphs recorded,
 * out4[2] recordings that failed (those calls ran directly), out4[3] calls
 * that enqueued their kernels directly (first sightings, debug outputs,
 * calls on a capturing stream).  out4 is host memory of 4 entries. */
void moe_cache_stats(unsigned long long *out4);

/* Synchronises `stream`, returns the first device-side error recorded in the
 * workspace since the last call (MOE_OK if none) and clears it.  *info_out
 * (may be NULL) receives where it happened. */
moe_status_t moe_get_status(void *workspace, void *stream, uint32_t *info_out);

/* Static description of a status code. */
const char *moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
