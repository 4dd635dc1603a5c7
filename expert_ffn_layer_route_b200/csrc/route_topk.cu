// Router product and top-k selection with renormalised softmax gates.
//
// The router is the dense per-token scoring that "picks a few" experts
// ("Mixture of experts VRAM: total vs active parameters", section "How current
// MoE models route each token"); every token goes to a fixed number k of
// experts (same section).  Selection is on the logits (softmax is monotone),
// largest first, the lower expert index winning ties; the gates are the
// softmax of the selected logits, which equals the softmax over all E experts
// renormalised over the selection.
//
// Kernel 1 (router_logits_kernel): a block computes an 8-token x 4-expert tile
// of logits (1, 2 or 4 tokens when the batch is smaller).  Thread t of 256 owns the 8-element chunks t, t+256, ... of the
// hidden dimension, accumulates its products in fp32 in that order, then the
// partial sums are folded by a warp butterfly and the 8 warps are added in a
// fixed order.  Every logit - every expert column - goes through the same
// summation tree (depth MOE_ROUTER_SUM_DEPTH(d)), so identical router rows
// give bit-identical logits and ties resolve exactly.
//
// Kernel 2 (topk_kernel): one warp per token.  k rounds of a warp-wide
// argmax over (logit desc, index asc); gates from expf in fp32.
#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "route_device.cuh"

namespace moe {

template <bool kFp32Router, int kRouterTokens>
__global__ void __launch_bounds__(kRouterThreads)
    router_logits_kernel(const __nv_bfloat16* __restrict__ x, const void* __restrict__ wr,
                         const float* __restrict__ bias, float* __restrict__ logits, int T, int d, int E) {
  pdl_wait_and_trigger();
  __shared__ float part[(kRouterThreads / 32) * kRouterTokens * kRouterExperts];
  const int t0 = blockIdx.x * kRouterTokens;
  const int e0 = blockIdx.y * kRouterExperts;
  router_tile<kFp32Router, kRouterTokens>(x, wr, bias, T, d, E, t0, e0, part, [&](int a, int b, float v) {
    logits[(size_t)(t0 + a) * E + e0 + b] = v;
  });
}

__global__ void __launch_bounds__(256)
    topk_kernel(const float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                int T, int E, int k) {
  pdl_wait_and_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= T) return;
  topk_warp(logits + (size_t)warp * E, E, k, topk_idx + (size_t)warp * k, topk_w + (size_t)warp * k);
}

cudaError_t launch_route_topk(const moe_layer_desc& dsc, const void* x, const void* wr, const float* bias,
                              float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  const int T = dsc.T, d = dsc.d_model, E = dsc.n_experts, k = dsc.top_k;
  {
  // tokens per block: 8, or the batch rounded up to a power of two when
  // smaller (a block's thread keeps the same summation order either way)
  const int tok = T >= 8 ? 8 : (T > 2 ? 4 : T);
  auto go = [&](auto kern) {
    return launch_pdl(kern, dim3(ceil_div(T, tok), ceil_div(E, kRouterExperts)), dim3(kRouterThreads), 0, st,
                      static_cast<const __nv_bfloat16*>(x), wr, bias, logits, T, d, E);
  };
  ProfScope prof("router_logits", st);
  cudaError_t err;
  if (dsc.router_fp32)
    err = tok == 1 ? go(router_logits_kernel<true, 1>) : tok == 2 ? go(router_logits_kernel<true, 2>)
        : tok == 4 ? go(router_logits_kernel<true, 4>) : go(router_logits_kernel<true, 8>);
  else
    err = tok == 1 ? go(router_logits_kernel<false, 1>) : tok == 2 ? go(router_logits_kernel<false, 2>)
        : tok == 4 ? go(router_logits_kernel<false, 4>) : go(router_logits_kernel<false, 8>);
  if (err != cudaSuccess) return err;
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ProfScope prof("topk", st);
  return launch_pdl(topk_kernel, dim3(ceil_div(T * 32, 256)), dim3(256), 0, st, logits, topk_idx, topk_w, T, E, k);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Router + top-k for callers that cannot allocate device memory.
//
// moe_route_topk takes its logits scratch from a caller-provided workspace.
// Some callers have no way to provide one: plugins whose host framework owns
// every device allocation and hands them none, runtimes that fix their device
// memory at start-up and forbid allocation afterwards, code on paths where a
// device allocation would synchronise or fail.  For them the logits live in a
// fixed file-scope device array instead, sized for T * n_experts <= 262144
// (1 MiB of fp32); every GPU that loads this library holds it until exit.
//
// Host code must not pass the array's name to a kernel: on the host it is a
// stand-in symbol, not a device address.  The device address is looked up
// with cudaGetSymbolAddress on the first call made with a device current, and
// again whenever the context current on that device has changed since (the
// array is reloaded at a new address in a new context, e.g. after
// cudaDeviceReset), so that a first call should come before any stream
// capture.  All calls share the one array: calls that overlap on the GPU
// (different streams, no ordering between them) race on it.  Nothing in it
// needs to start at zero: each call writes every logit it later reads.
namespace {

constexpr size_t kNoAllocLogitsMax = 262144;
__device__ __align__(256) float g_noalloc_logits[kNoAllocLogitsMax];

constexpr int kNoAllocMaxDevices = 64;
struct NoAllocSlot {
  uintptr_t ctx;  // context the address was looked up in
  float* ptr;
};
std::mutex g_noalloc_mu;
NoAllocSlot g_noalloc[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" moe_status moe_route_topk_noalloc(const moe_layer_desc* desc, const void* x, const void* w_router,
                                             const float* logit_bias, int32_t* topk_idx, float* topk_w,
                                             void* stream) {
  size_t ws_bytes = 0;
  moe_status s = moe_workspace_size(desc, &ws_bytes);  // validates the descriptor
  if (s != MOE_OK) return s;
  if (desc->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router)) & 15u) return MOE_ERR_INVALID_ARG;
  if ((size_t)desc->T * (size_t)desc->n_experts > kNoAllocLogitsMax) return MOE_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
  float* logits = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSlot& slot = g_noalloc[dev];
    const uintptr_t ctx = moe::current_ctx();  // 0 before the runtime made a context on this thread
    if (!slot.ptr || ctx == 0 || slot.ctx != ctx) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_logits) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
      slot.ptr = static_cast<float*>(p);
      slot.ctx = moe::current_ctx();
    }
    logits = slot.ptr;
  }
  return moe::launch_route_topk(*desc, x, w_router, logit_bias, logits, topk_idx, topk_w,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
