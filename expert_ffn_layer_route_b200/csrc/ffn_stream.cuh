// Argument block and launcher of the weight-streaming grouped FFN kernel.
#pragma once

#include "common.cuh"
#include "tmap.cuh"

namespace moe {

enum Fmt : int { kBF16 = MOE_W_BF16, kMXFP4 = MOE_W_MXFP4, kNVFP4 = MOE_W_NVFP4, kINT4 = MOE_W_INT4_G128 };

struct alignas(64) FfnArgs {
  // TMA maps: routed weights [n_phys][rows][row bytes], shared weights
  // [n_shared][rows][row bytes], activation rows [rows_total][K*2 bytes]
  CUtensorMap tm_w;
  CUtensorMap tm_wsh;
  CUtensorMap tm_x;
  // block scales (1-D bulk copies per item)
  const uint8_t* s;
  int64_t stride_s;
  const uint8_t* s_sh;
  int64_t stride_s_sh;
  const float* gsc;     // NVFP4 global scales [E]
  const float* gsc_sh;  // [n_shared]
  const int32_t* slot_map;
  int n_phys;
  int n_shared;
  // problem
  int E, T, k;
  int N;  // output rows: d_ff (stage 1 gate rows; up rows follow at +d_ff) or d (stage 2)
  int K;  // reduction length
  const int32_t* offsets;  // [E+1]
  const int32_t* xexp;     // per activation row power-of-two exponent (4-bit formats)
  const float* xbias;      // INT4: per activation row and 128-group, the constant part
                           // 1032 sum(even x) + 1152 sum(odd x') of the offset decode
  // outputs (bf16): stage 1 writes rows [rows_total][d_ff]; stage 2 writes routed
  // rows to out_routed [T*k][d] and shared rows to out_shared [n_shared][T][d]
  __nv_bfloat16* out_routed;
  __nv_bfloat16* out_shared;
  int n_stages;
  int n_sslots;    // ring stages that carry one item's block scales (1, 2, 4 or 8)
  int tmem_cols;   // TMEM columns holding one weight row's block scales
  int tmem_alloc;  // TMEM columns allocated per block (power of two >= 32)
  int w_l2_first;        // 1: weight boxes marked evict-first in L2; 0 (default): normal priority
  int32_t* work_ctr;     // launch-wide item counter, zero before the launch
  // Split K: each item's K chunks in `split` consecutive slices, one work
  // item each; every consumer warp stores its fp32 partial accumulators, and
  // the warp that arrives last (per-item, per-warp counters, zero before the
  // launch) sums the slices in slice order and runs the epilogue.
  int split;             // slices per item (1: no split; set by the launcher)
  int split_cap;         // work items the buffers below hold (0: split off)
  int32_t* split_ctr;    // [split_cap][consumer warps] arrivals
  float* split_part;     // [split_cap][consumer threads][8] fp32 partials
};

// Capacity of the split-K buffers (work items), and their sizes in bytes.
constexpr int kStreamSplitCap = 512;
constexpr int kStreamSplitCtrInts = kStreamSplitCap * 8;
constexpr size_t kStreamSplitPartBytes = (size_t)kStreamSplitCap * 256 * 8 * sizeof(float);

// Launch one stage (gate_up: stage 1 with SwiGLU; else stage 2) of the
// streaming FFN.  The caller fills everything but the tensor maps, which are
// encoded here from the raw pointers.  Sets *unsupported when the
// shared-memory plan cannot fit.
struct FfnPointers {
  const void* w;       // routed weights base
  int64_t stride_w;    // bytes between experts
  const void* w_sh;    // shared weights base (or null)
  int64_t stride_w_sh;
  const void* x;       // activation rows [rows_total][K] (f16 or bf16)
  int rows_total;
};

cudaError_t launch_ffn_stream(int F, bool gate_up, FfnArgs a, const FfnPointers& p, int T, int n_sms,
                              int smem_max, int smem_per_sm, cudaStream_t st, int* unsupported);

}  // namespace moe
