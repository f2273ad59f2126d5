// moe_route_static: the router with its scratch in a fixed device array, for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not available or not
// allowed -- for instance a plug-in hosted by an inference runtime that owns
// all device memory and hands out no allocator, or a hot loop whose
// allocation policy forbids growing memory after start-up.  Such callers can
// still pass their own input and output buffers, but not a workspace.
//
// The scratch lives in one file-scope __device__ array of kRouteStaticBytes
// (8 MiB).  Every GPU on which this library's module is loaded holds that
// array until the process exits.  Its device address is looked up once per
// device with cudaGetSymbolAddress (host code cannot use the array's name as
// a device pointer); the first call on each device does that lookup, so make
// the first call on a device outside any stream capture.  All calls share the
// one array: two calls whose kernels overlap on the GPU (different streams,
// or different host threads) race on it and must be serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {
namespace {

constexpr size_t kRouteStaticBytes = size_t(8) << 20;
constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kRouteStaticBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxStaticDevices] = {};

// Regions carved from the static array (1024-byte aligned, like the workspace).
struct StaticRouteLayout {
  size_t header, logits, xnorm, wnorm, amax_tok, cand, total;
};

StaticRouteLayout static_route_layout(int T, int E) {
  StaticRouteLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.header = take(kStatusBytes);
  L.logits = take(static_cast<size_t>(T) * E * 4);
  L.xnorm = take(static_cast<size_t>(T) * 4);
  L.wnorm = take(static_cast<size_t>(E) * 4);
  L.amax_tok = take(static_cast<size_t>(T) * 4);
  L.cand = take(static_cast<size_t>(T) * E * 16);
  L.total = off;
  return L;
}

// Device address of the static scratch on the current device (looked up once).
moe_status_t static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxStaticDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_route_static(const void* hidden, const void* router_w,
                                         const float* router_bias, int T, int H, int E, int top_k,
                                         int32_t* topk_ids, float* topk_w, void* stream) {
  if (E < 1 || E > kMaxExperts || top_k < 1 || top_k > E || top_k > kMaxTopK)
    return MOE_ERR_INVALID_ARG;
  if (T < 1 || H < 128 || H > 8192 || H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!hidden || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) & 15u) || (reinterpret_cast<uintptr_t>(router_w) & 15u) ||
      (reinterpret_cast<uintptr_t>(router_bias) & 3u))   // the bias is read as fp32
    return MOE_ERR_MISALIGNED;
  if (static_cast<long long>(T) * E > (1LL << 24)) return MOE_ERR_EXCEEDS_STATIC_SCRATCH;
  const StaticRouteLayout L = static_route_layout(T, E);
  if (L.total > kRouteStaticBytes) return MOE_ERR_EXCEEDS_STATIC_SCRATCH;
  void* base = nullptr;
  moe_status_t s = static_scratch(&base);
  if (s != MOE_OK) return s;
  char* b = static_cast<char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // only the header (status / counters) must start at zero; every other
  // region is written before it is read within the call
  if (cudaMemsetAsync(b + L.header, 0, kStatusBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
  RouterArgs ra{static_cast<const __nv_bfloat16*>(hidden), static_cast<const __nv_bfloat16*>(router_w),
                router_bias, T, H, E, top_k,
                reinterpret_cast<float*>(b + L.logits), reinterpret_cast<float*>(b + L.xnorm),
                reinterpret_cast<float*>(b + L.wnorm), reinterpret_cast<float*>(b + L.amax_tok),
                topk_ids, topk_w, reinterpret_cast<unsigned char*>(b + L.cand),
                reinterpret_cast<uint32_t*>(b + L.header), nullptr};
  return launch_router(ra, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
