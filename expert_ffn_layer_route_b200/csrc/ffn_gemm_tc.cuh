// Argument block and launcher of the tcgen05 grouped-GEMM FFN (prefill path).
#pragma once

#include "ffn_stream.cuh"

namespace moe {

struct alignas(64) GemmArgs {
  CUtensorMap tm_a;    // activation rows [rows_total][K] bf16 (as bytes)
  CUtensorMap tm_b;    // routed weights [n_phys][rows][K] bf16
  CUtensorMap tm_bsh;  // shared weights [n_shared][rows][K] bf16
  const int32_t* offsets;
  const int32_t* slot_map;
  int n_phys;
  int n_shared;
  int E, T, k;
  int N;  // stage 1: d_ff (gate rows; up rows follow at +d_ff); stage 2: d
  int K;
  __nv_bfloat16* out_routed;  // stage 1: h [rows_total][d_ff]; stage 2: y [T*k][d]
  __nv_bfloat16* out_shared;  // stage 2: [n_shared][T][d]
};

using GemmPointers = FfnPointers;

// True when the tensor-core GEMM path handles this stage (bf16 weights, K a
// multiple of 64, N a multiple of the tile).
bool gemm_path_supported(int F, int N, int K, bool gate_up);

cudaError_t launch_ffn_gemm(bool gate_up, GemmArgs a, const GemmPointers& p, int n_sms, int smem_max,
                            cudaStream_t st, int* unsupported);

}  // namespace moe
