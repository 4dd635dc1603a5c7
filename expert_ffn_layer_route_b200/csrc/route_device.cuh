// Device routines shared by the routing kernels and the fused small-batch
// routing kernel, so that both compute bit-identical results:
//   router_tile  - a kTok-token x 4-expert tile of router logits (fixed fp32
//                  summation tree, depth MOE_ROUTER_SUM_DEPTH(d));
//   topk_warp    - one token's top-k over its E logits and the renormalised
//                  softmax gates, by one warp;
//   prep_row     - one activation row into the grouped FFN's input format.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kRouterExperts = 4;  // experts per tile
constexpr int kRouterThreads = 256;

// logits of tokens [t0, t0 + kTok) x experts [e0, e0 + kExp) (clipped to T,
// E).  Thread t of 256 owns the 8-element chunks t, t+256, ... of the hidden
// dimension, accumulates its products in fp32 in that order, the partial sums
// are folded by a warp butterfly and the 8 warps are added in a fixed order;
// a logit's summation tree depends neither on kTok nor on kExp.  `part` is
// 8 x (kTok * kExp) floats of shared memory (kTok * kExp <= 256).  Calls
// store(a, b, v) from thread a * kExp + b for each token a < nt and expert
// b < ne of the tile.  All 256 threads of the block must call it (it
// synchronises the block).
template <bool kFp32Router, int kTok, int kExp = kRouterExperts, typename Store>
__device__ __forceinline__ void router_tile(const __nv_bfloat16* __restrict__ x, const void* __restrict__ wr,
                                            const float* __restrict__ bias, int T, int d, int E, int t0, int e0,
                                            float* part, Store store) {
  static_assert(kTok * kExp <= kRouterThreads, "one folding thread per logit");
  const int tid = threadIdx.x;
  const int nt = min(kTok, T - t0);
  const int ne = min(kExp, E - e0);
  float acc[kTok][kExp];
#pragma unroll
  for (int a = 0; a < kTok; ++a)
#pragma unroll
    for (int b = 0; b < kExp; ++b) acc[a][b] = 0.f;

  // Per chunk every accumulator adds its 8 products in q order; the loop
  // nest around that (which operand is held in registers while the other
  // streams) changes no sum.  Few experts per tile: the experts' weights are
  // held and the tokens stream; many (small batches): the tokens are held.
  const int nchunk = d / 8;
  auto load_w = [&](int e, int c, float (&wv)[8]) {
    if constexpr (kFp32Router) {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(wr) + (size_t)e * d + c * 8);
      float4 u0 = __ldg(p), u1 = __ldg(p + 1);
      wv[0] = u0.x; wv[1] = u0.y; wv[2] = u0.z; wv[3] = u0.w;
      wv[4] = u1.x; wv[5] = u1.y; wv[6] = u1.z; wv[7] = u1.w;
    } else {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(wr) + (size_t)e * d + c * 8));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        wv[2 * q] = bf16_bits_to_f32(w4[q] & 0xffffu);
        wv[2 * q + 1] = bf16_bits_to_f32(w4[q] >> 16);
      }
    }
  };
  auto load_x = [&](int a, int c, float (&xv)[8]) {
    const int t = t0 + (a < nt ? a : 0);
    uint4 u = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d + c * 8));
    const uint32_t x4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xv[2 * q] = bf16_bits_to_f32(x4[q] & 0xffffu);
      xv[2 * q + 1] = bf16_bits_to_f32(x4[q] >> 16);
    }
  };
  for (int c = tid; c < nchunk; c += kRouterThreads) {
    if constexpr (kExp <= kRouterExperts) {
      float wv[kExp][8];
#pragma unroll
      for (int b = 0; b < kExp; ++b) load_w(e0 + (b < ne ? b : 0), c, wv[b]);
#pragma unroll
      for (int a = 0; a < kTok; ++a) {
        float xv[8];
        load_x(a, c, xv);
#pragma unroll
        for (int b = 0; b < kExp; ++b)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(xv[q], wv[b][q]));
      }
    } else {
      float xv[kTok][8];
#pragma unroll
      for (int a = 0; a < kTok; ++a) load_x(a, c, xv[a]);
#pragma unroll
      for (int b = 0; b < kExp; ++b) {
        float wv[8];
        load_w(e0 + (b < ne ? b : 0), c, wv);
#pragma unroll
        for (int a = 0; a < kTok; ++a)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(xv[a][q], wv[q]));
      }
    }
  }
  // warp butterfly (identical association in every lane and every column)
#pragma unroll
  for (int a = 0; a < kTok; ++a)
#pragma unroll
    for (int b = 0; b < kExp; ++b)
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc[a][b] = __fadd_rn(acc[a][b], __shfl_xor_sync(0xffffffffu, acc[a][b], off));

  const int warp = tid >> 5, lane = tid & 31;
  constexpr int kCols = kTok * kExp;
  if (lane == 0) {
#pragma unroll
    for (int a = 0; a < kTok; ++a)
#pragma unroll
      for (int b = 0; b < kExp; ++b) part[warp * kCols + a * kExp + b] = acc[a][b];
  }
  __syncthreads();
  if (tid < kCols) {
    const int a = tid / kExp, b = tid % kExp;
    float s = part[tid];
#pragma unroll
    for (int w = 1; w < kRouterThreads / 32; ++w) s = __fadd_rn(s, part[w * kCols + tid]);
    if (a < nt && b < ne) {
      if (bias != nullptr) s = __fadd_rn(s, __ldg(bias + e0 + b));
      store(a, b, s);
    }
  }
  __syncthreads();  // `part` may be reused by the next tile
}

// (value, index) ordering: larger value first, then lower index.  NaN never wins.
__device__ __forceinline__ bool topk_beats(float v, int i, float w, int j) {
  return (v > w) || (v == w && i < j);
}

// One token: k rounds of a warp-wide argmax over (logit desc, index asc) of
// its E logits `lt` (global or shared memory); gates = softmax of the
// selected logits (exp in fp32).  Lane j < k writes pick j to idx_out[j] /
// w_out[j].  Every lane of the warp must call it.
__device__ __forceinline__ void topk_warp(const float* lt, int E, int k, int32_t* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  int prev_i = -1;
  float prev_v = __int_as_float(0x7f800000);  // +inf: everything is below the previous pick
  float my_v = 0.f;
  int my_i = -1;
  for (int j = 0; j < k; ++j) {
    // best element strictly after (prev_v, prev_i) in the total order
    float bv = __int_as_float(0xff800000);  // -inf
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = lt[e];
      if (v != v) continue;  // NaN is never selected
      if (!topk_beats(prev_v, prev_i, v, e)) continue;
      if (topk_beats(v, e, bv, bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (topk_beats(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (bi == 0x7fffffff || bi < 0 || bi >= E) {
      bi = -1;
      if (lane == 0) set_status(MOE_ERR_DEVICE_INDEX);
    }
    if (lane == j) { my_v = bv; my_i = bi; }
    prev_v = bv;
    prev_i = bi;
  }
  // gates: softmax over the selected logits (lane j holds pick j; pick 0 is the max)
  const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = (lane < k) ? expf(my_v - vmax) : 0.f;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(0xffffffffu, ex, j));
  if (lane < k) {
    idx_out[lane] = my_i;
    w_out[lane] = ex / sum;
  }
}

enum PrepMode : int { kF16 = 0, kF16Int4 = 1, kCopyBf16 = 2 };

// One activation row of K values (src; nullptr: a row without source, written
// as zeros) into the grouped FFN's input format, by threads tid of nth (nth a
// multiple of 32, at most 1024; every thread of the group must call it):
//   kCopyBf16: the bf16 row as is;
//   kF16:      fp16 after scaling by 2^-p, p = floor(log2(max|row|)) - 14, so
//              that the largest magnitude lies in [2^14, 2^15); *rexp = p;
//   kF16Int4:  as kF16, with the odd-K values divided by 16, each 8-element
//              group stored in the order 0,4,1,5,2,6,3,7 (the INT4 decoder's
//              pairing), and per 128-wide scale group g
//              gbias[g] = 1032 sum_even h + 1152 sum_odd h over the stored fp16
//              values h (summed in fp64, rounded once to fp32).
// `red` is nth / 32 floats of shared memory.  The fp64 group sums reduce the
// same 16 chunks in the same butterfly order for any nth that is a multiple
// of 16, so the result does not depend on the thread count.  kWarp: the group
// is one warp (nth = 32, tid = lane); no block barrier, `red` unused.
template <int kMode, bool kWarp = false>
__device__ __forceinline__ void prep_row(const __nv_bfloat16* __restrict__ src, int K, void* __restrict__ dst,
                                         int32_t* rexp, float* gbias, int tid, int nth, float* red) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  const bool have = src != nullptr;
  const int nchunk = K / 8;
  if constexpr (kMode == kCopyBf16) {
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int c = tid; c < nchunk; c += nth) d[c] = have ? __ldg(s + c) : z4;
    return;
  }
  float amax = 0.f;
  for (int c = tid; c < nchunk; c += nth) {
    const uint4 u = have ? __ldg(s + c) : z4;
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[q] & 0xffffu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[q] >> 16)));
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if constexpr (!kWarp) {
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    // (callers synchronise the thread group with a block barrier: nth is the block or a whole-block subset)
    __syncthreads();
    amax = red[0];
    for (int w = 1; w < nth / 32; ++w) amax = fmaxf(amax, red[w]);
    __syncthreads();  // red may be reused by the next row
  }
  int p = 0;
  if (amax > 0.f && amax <= 3.0e38f) {
    int ex;
    frexpf(amax, &ex);  // amax = m * 2^ex, m in [0.5, 1)
    p = ex - 15;        // floor(log2(amax)) - 14
  }
  if (tid == 0) *rexp = p;
  const float scale = ldexpf(1.f, -p);
  uint4* d = reinterpret_cast<uint4*>(dst);
  // every thread runs the same number of rounds so that the 16-lane group
  // sums below see full warps (nchunk is a multiple of 16 for INT4)
  for (int base = 0; base < nchunk; base += nth) {
    const int c = base + tid;
    const bool on = c < nchunk;
    float f[8];
    if (on) {
      const uint4 u = have ? __ldg(s + c) : z4;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f[2 * q] = bf16_bits_to_f32(w[q] & 0xffffu) * scale;
        f[2 * q + 1] = bf16_bits_to_f32(w[q] >> 16) * scale;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] = 0.f;
    }
    __half h[8];
    if constexpr (kMode == kF16Int4) {
      const int order[8] = {0, 4, 1, 5, 2, 6, 3, 7};
      double even = 0.0, odd = 0.0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int kk = order[q];
        h[q] = __float2half_rn((kk & 1) ? f[kk] * 0.0625f : f[kk]);
        if (kk & 1) odd += (double)__half2float(h[q]); else even += (double)__half2float(h[q]);
      }
      double part = 1032.0 * even + 1152.0 * odd;
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (on && (tid & 15) == 0) gbias[c >> 4] = (float)part;
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) h[q] = __float2half_rn(f[q]);
    }
    if (on) d[c] = *reinterpret_cast<uint4*>(h);
  }
}

}  // namespace moe
