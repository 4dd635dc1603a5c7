// Routing and activation preparation of a small batch (T <= 8 tokens) in one
// launch.
//
// A decode step of a few tokens spends most of its time on fixed per-kernel
// latency, not on bytes (the router, top-k, permutation and activation-prep
// kernels each read a few KB to MB).  This kernel does all four as one
// thread-block cluster:
//   1. every CTA brings its slice of the router weights into L2 before the
//      dependent-launch wait, then computes the logits of its experts for
//      all T tokens (the router tile of the standalone router kernel: the
//      same fp32 summation tree, so the same logits) and stores them into
//      CTA 0's shared memory through distributed shared memory;
//   2. CTA 0 selects each token's top-k with renormalised softmax gates (one
//      warp per token, the standalone top-k routine) and forms the stable
//      per-expert permutation by counting (offsets, row of each (token, slot)
//      pair, token of each row; rows of one expert in ascending token order);
//   3. the activation rows in expert order, in the grouped FFN's input format
//      (the standalone prep routine): one CTA per row when the rows fit the
//      cluster, else one warp per row.
// The steps are ordered by cluster barriers, which the hardware schedules
// together, so no counter or flag is polled.  The router step follows "a
// router that picks a few of them per token" ("Mixture of experts VRAM:
// total vs active parameters", section "How current MoE models route each
// token"); the grouping follows "Understanding MoE Inference Costs on
// Galactus", section "Prompt processing is a different phase".
#include <cooperative_groups.h>

#include <atomic>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "route_device.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kSmallMaxT = 8;
constexpr int kSmallMaxPairs = 64;
// logits per router tile: 32 experts for one token, 4 for eight
constexpr int kSmallTileLogits = 32;
// experts per router tile for kTok tokens: at most 16, so that a CTA's slice
// of 128 experts / 8 CTAs fills its tile without padding columns
__host__ __device__ constexpr int small_tile_experts(int tok) {
  return kSmallTileLogits / tok < 16 ? kSmallTileLogits / tok : 16;
}

struct RouteSmallArgs {
  const __nv_bfloat16* x;
  const void* wr;
  const float* bias;
  int T, d, E, k, n_shared;
  int e_per_cta;  // experts per CTA (a multiple of 4)
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;
  int32_t* row_token;
  int32_t* inv;
  void* xperm;
  int32_t* xexp;
  float* gbias;
  int32_t* zero;  // counters the FFN stages start from
  int n_zero;
};

// Shared memory (floats, then ints): router partials [8][32], row-max
// scratch [8], all logits [kTok][E] (written into CTA 0's copy by every CTA),
// the gates [64], the picks [64], the rows' tokens [64] (CTA 0) and this
// CTA's copy of them [64].
__host__ __device__ constexpr int small_smem_words(int tok, int E) {
  return 8 * kSmallTileLogits + 8 + tok * E + 4 * kSmallMaxPairs;
}

}  // namespace

template <bool kFp32Router, int kTok, int kMode>
__global__ void __launch_bounds__(kRouterThreads) route_prep_small_kernel(const __grid_constant__ RouteSmallArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int csize = (int)cluster.num_blocks();
  const int tid = threadIdx.x, warp = tid >> 5;
  extern __shared__ float smem_f[];
  constexpr int kSmallExp = small_tile_experts(kTok);  // experts per router tile
  float* s_part = smem_f;                      // [8 * kSmallTileLogits]
  float* s_red = s_part + 8 * kSmallTileLogits;  // [8]
  float* s_all = s_red + 8;                    // [kTok][E], filled on CTA 0
  float* s_w = s_all + kTok * a.E;             // CTA 0: [64]
  int* s_idx = reinterpret_cast<int*>(s_w + kSmallMaxPairs);  // CTA 0: [64]
  int* s_rtok = s_idx + kSmallMaxPairs;        // CTA 0: [64]
  int* s_rl = s_rtok + kSmallMaxPairs;         // [64], this CTA's copy of s_rtok
  const int T = a.T, E = a.E, k = a.k, R = T * k;
  const int e_lo = rank * a.e_per_cta;
  const int e_hi = min(E, e_lo + a.e_per_cta);

  // The router weights are not written by the kernels this one may overlap
  // (programmatic dependent launch): bring this CTA's slice into L2 while the
  // predecessor finishes.
  if (e_hi > e_lo) {
    const size_t esz = kFp32Router ? 4 : 2;
    const char* w0 = static_cast<const char*>(a.wr) + (size_t)e_lo * a.d * esz;
    const size_t nbytes = (size_t)(e_hi - e_lo) * a.d * esz;
    for (size_t o = (size_t)tid * 128; o < nbytes; o += (size_t)kRouterThreads * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(w0 + o));
  }
  pdl_wait_and_trigger();
  for (int i = rank * kRouterThreads + tid; i < a.n_zero; i += csize * kRouterThreads) a.zero[i] = 0;
  // 1. router logits of this CTA's experts, stored into CTA 0's table
  float* s_all0 = cluster.map_shared_rank(s_all, 0);
  for (int e0 = e_lo; e0 < e_hi; e0 += kSmallExp) {
    router_tile<kFp32Router, kTok, kSmallExp>(a.x, a.wr, a.bias, T, a.d, e_hi, 0, e0, s_part,
                                              [&](int t, int b, float v) { s_all0[t * E + e0 + b] = v; });
  }
  if (rank == 0)
    for (int i = tid; i < R; i += kRouterThreads) s_rtok[i] = -1;
  cluster.sync();
  // 2. CTA 0: top-k + gates per token, then the stable permutation by counting:
  //    the row of pair i is the number of valid pairs with a smaller expert
  //    plus the earlier pairs of its own expert; offsets[e] counts the valid
  //    pairs with an expert below e
  if (rank == 0) {
    if (warp < T) topk_warp(s_all + warp * E, E, k, s_idx + warp * k, s_w + warp * k);
    __syncthreads();
    for (int i = tid; i < R; i += kRouterThreads) {
      const int e = s_idx[i];
      a.topk_idx[i] = e;
      a.topk_w[i] = s_w[i];
      if (e < 0 || e >= E) {
        set_status(MOE_ERR_DEVICE_INDEX);
        a.inv[i] = -1;
        continue;
      }
      int r = 0;
      for (int j = 0; j < R; ++j) {
        const int f = s_idx[j];
        r += ((unsigned)f < (unsigned)e || (f == e && j < i)) ? 1 : 0;
      }
      s_rtok[r] = i / k;
      a.row_token[r] = i / k;
      a.inv[i] = r;
    }
    for (int e = tid; e <= E; e += kRouterThreads) {
      int c = 0;
      for (int j = 0; j < R; ++j) c += (unsigned)s_idx[j] < (unsigned)e ? 1 : 0;
      a.offsets[e] = c;
    }
  }
  cluster.sync();
  // 3. activation rows in expert order: routed rows, then every token once per
  //    shared expert.  CTA 0's row tokens are copied first, after which the
  //    CTA signals that it no longer reads CTA 0's shared memory; it waits for
  //    the others' signals only before exiting.
  const int* rtok0 = cluster.map_shared_rank(s_rtok, 0);
  for (int i = tid; i < R; i += kRouterThreads) s_rl[i] = rtok0[i];
  __syncthreads();
  cluster.barrier_arrive();
  // one CTA per row when the rows fit the cluster, else one warp per row
  // (both group sizes give the same row: see prep_row)
  const int RT = R + a.n_shared * T;
  auto row_src = [&](int r) -> const __nv_bfloat16* {
    const int srow = r < R ? s_rl[r] : (r - R) % T;
    return (unsigned)srow < (unsigned)T ? a.x + (size_t)srow * a.d : nullptr;  // a dropped pair's row: zeros
  };
  auto row_dst = [&](int r) { return static_cast<uint8_t*>(a.xperm) + (size_t)r * a.d * 2; };
  if (RT <= csize) {
    if (rank < RT)
      prep_row<kMode>(row_src(rank), a.d, row_dst(rank), a.xexp ? a.xexp + rank : nullptr,
                      a.gbias ? a.gbias + (size_t)rank * (a.d / 128) : nullptr, tid, kRouterThreads, s_red);
  } else {
    const int nwarps = csize * (kRouterThreads / 32);
    for (int r = rank * (kRouterThreads / 32) + warp; r < RT; r += nwarps)
      prep_row<kMode, true>(row_src(r), a.d, row_dst(r), a.xexp ? a.xexp + r : nullptr,
                            a.gbias ? a.gbias + (size_t)r * (a.d / 128) : nullptr, tid & 31, 32, nullptr);
  }
  cluster.barrier_wait();  // CTA 0's shared memory stays until every CTA has read it
}

// ------------------------------------------------------------------ host side
namespace {

// Non-portable cluster sizes (16) need a per-kernel attribute, set once per
// device and context.
template <auto Kern>
cudaError_t allow_cluster16_once() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static uintptr_t done[kMaxDev] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lk(mu);
  const uintptr_t ctx = current_ctx();
  if (dev >= 0 && dev < kMaxDev && ctx != 0 && done[dev] == ctx) return cudaSuccess;
  err = cudaFuncSetAttribute(Kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (err != cudaSuccess) return err;
  if (dev >= 0 && dev < kMaxDev) done[dev] = current_ctx();
  return cudaSuccess;
}

template <bool F32, int TOK, int MODE>
cudaError_t launch_small(RouteSmallArgs a, cudaStream_t st) {
  auto kern = route_prep_small_kernel<F32, TOK, MODE>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kRouterThreads);
  cfg.stream = st;
  cfg.attrs = attr;
  // 8 CTAs, 16 for more than 256 experts when the device can co-schedule a
  // cluster of 16 (a non-portable size); a multiple of 4 experts per CTA
  int csize = 8;
  size_t smem = 0;
  cudaError_t err;
  for (int want = a.E > 256 ? 16 : 8; want >= 8; want /= 2) {
    csize = want;
    a.e_per_cta = ((ceil_div(a.E, csize) + 3) / 4) * 4;
    smem = (size_t)small_smem_words(TOK, a.E) * 4;
    if ((err = set_dyn_smem_once<route_prep_small_kernel<F32, TOK, MODE>>(smem)) != cudaSuccess) return err;
    if (csize == 8) break;
    if (allow_cluster16_once<route_prep_small_kernel<F32, TOK, MODE>>() != cudaSuccess) {
      (void)cudaGetLastError();
      continue;
    }
    // the occupancy answer, asked once per kernel and device
    constexpr int kMaxDev = 64;
    static std::atomic<int> fits16_dev[kMaxDev];  // 0: not asked, 1: no, 2: yes
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
      (void)cudaGetLastError();
      dev = 0;
    }
    std::atomic<int>& fits16 = fits16_dev[dev];
    if (fits16.load() == 0) {
      cfg.gridDim = dim3(csize);
      cfg.dynamicSmemBytes = smem;
      attr[0].val.clusterDim.x = csize;
      cfg.numAttrs = 1;
      int n_clusters = 0;
      const bool ok = cudaOccupancyMaxActiveClusters(&n_clusters, kern, &cfg) == cudaSuccess && n_clusters > 0;
      if (!ok) (void)cudaGetLastError();
      fits16.store(ok ? 2 : 1);
    }
    if (fits16.load() == 2) break;
  }
  cfg.gridDim = dim3(csize);
  cfg.dynamicSmemBytes = smem;
  attr[0].val.clusterDim.x = csize;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  ProfScope prof("route_prep_small", st);
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool F32, int TOK>
cudaError_t launch_small_mode(int mode, const RouteSmallArgs& a, cudaStream_t st) {
  switch (mode) {
    case kF16: return launch_small<F32, TOK, kF16>(a, st);
    case kF16Int4: return launch_small<F32, TOK, kF16Int4>(a, st);
    default: return launch_small<F32, TOK, kCopyBf16>(a, st);
  }
}

}  // namespace

// Used by default where one launch beats the four it replaces: batches of at
// most 4 tokens whose router fits one tile per CTA (at most min(16, 32 / tile-tokens)
// experts per CTA of 8).  Measured on B200, the gpt-oss-shaped layer (128
// experts, d = 2880) at T = 1 takes 52.5-54.8 us per layer fused vs 54.5-56.2
// unfused; the Kimi-shaped layer (384 experts, d = 7168) runs its router
// slices as 6 serial tiles on 16 SMs and loses (T = 1: 109.6 vs 103.8 us;
// T = 8: 317.7 vs 289.1 us), as does T = 8 with 128 experts (123.6 vs
// 118.2 us), where the cluster waits for 8 free SMs of one GPC while the
// previous kernel drains.  MOE_FUSED_ROUTE=1 / 0 forces it on (within the
// kernel's limits) / off.
bool route_prep_small_supported(const moe_layer_desc& d) {
  const bool fits = d.T >= 1 && d.T <= kSmallMaxT && d.T * d.top_k <= kSmallMaxPairs && d.n_experts <= 1024 &&
                    d.d_model % 8 == 0;
  if (const char* e = std::getenv("MOE_FUSED_ROUTE")) {
    if (e[0] == '0') return false;
    if (e[0] == '1') return fits;
  }
  const int tok = d.T > 4 ? 8 : (d.T > 2 ? 4 : d.T);
  const int e_per_cta = ((ceil_div(d.n_experts, 8) + 3) / 4) * 4;
  return fits && d.T <= 4 && e_per_cta <= small_tile_experts(tok);
}

cudaError_t launch_route_prep_small(const moe_layer_desc& dsc, const void* x, const void* wr, const float* bias,
                                    int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* row_token,
                                    int32_t* inv, int mode, void* xperm, int32_t* xexp, float* gbias, int32_t* zero,
                                    int n_zero, cudaStream_t st) {
  RouteSmallArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.wr = wr;
  a.bias = bias;
  a.T = dsc.T;
  a.d = dsc.d_model;
  a.E = dsc.n_experts;
  a.k = dsc.top_k;
  a.n_shared = dsc.n_shared;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.offsets = offsets;
  a.row_token = row_token;
  a.inv = inv;
  a.xperm = xperm;
  a.xexp = xexp;
  a.gbias = gbias;
  a.zero = zero;
  a.n_zero = n_zero;
  // one tile covers every token (a logit's summation order does not depend on the tile width)
  const int tok = dsc.T > 4 ? 8 : (dsc.T > 2 ? 4 : dsc.T);
  const bool f32 = dsc.router_fp32 != 0;
  switch (tok) {
    case 1: return f32 ? launch_small_mode<true, 1>(mode, a, st) : launch_small_mode<false, 1>(mode, a, st);
    case 2: return f32 ? launch_small_mode<true, 2>(mode, a, st) : launch_small_mode<false, 2>(mode, a, st);
    case 4: return f32 ? launch_small_mode<true, 4>(mode, a, st) : launch_small_mode<false, 4>(mode, a, st);
    default: return f32 ? launch_small_mode<true, 8>(mode, a, st) : launch_small_mode<false, 8>(mode, a, st);
  }
}

}  // namespace moe
