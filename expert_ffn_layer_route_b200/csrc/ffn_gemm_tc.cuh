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

// 4-bit experts on the tensor cores (csrc/ffn_gemm_q4.cu): weights decoded to
// 16-bit values in shared memory once per (256-row activation block, weight
// tile), tcgen05.mma kind::f16 with fp32 accumulation.
struct alignas(64) GemmQ4Args {
  CUtensorMap tm_a;    // activation rows [rows_total][K] (bf16 for MXFP4, scaled fp16 otherwise), as bytes
  CUtensorMap tm_w;    // routed codes [n_phys][rows][K/2]
  CUtensorMap tm_wsh;  // shared codes [n_shared][rows][K/2]
  CUtensorMap tm_s;    // routed block scales [n_phys][rows][K/blk * scale bytes]
  CUtensorMap tm_ssh;  // shared block scales
  const int32_t* offsets;
  const int32_t* slot_map;
  int n_phys;
  int n_shared;
  int E, T, k;
  int N;  // stage 1: d_ff (gate rows; up rows follow at +d_ff); stage 2: d
  int K;
  const float* gsc;       // NVFP4 global scales [E] of this stage's matrix
  const float* gsc_sh;    // [n_shared]
  const int32_t* xexp;    // fp16 activations: per-row power of two to undo (NVFP4, INT4)
  __nv_bfloat16* out_routed;
  __nv_bfloat16* out_shared;
};

struct GemmQ4Pointers {
  const void* w;
  int64_t stride_w;
  const void* s;
  int64_t stride_s;
  const void* w_sh;
  int64_t stride_w_sh;
  const void* s_sh;
  int64_t stride_s_sh;
  const void* x;
  int rows_total;
};

// True when the 4-bit tensor-core path handles this stage: K a multiple of
// 64, the scale matrix's row a multiple of 16 bytes (K a multiple of 512 for
// MXFP4, 256 for NVFP4, 1024 for INT4), N a multiple of the tile.
bool gemm_q4_supported(int F, int N, int K, bool gate_up);
// MXFP4 multiplies bf16 activation rows; NVFP4 and INT4 fp16 rows scaled by a
// power of two per row.
bool gemm_q4_bf16_activations(int F);

cudaError_t launch_ffn_gemm_q4(int F, bool gate_up, GemmQ4Args a, const GemmQ4Pointers& p, int n_sms,
                               int smem_max, cudaStream_t st, int* unsupported);

}  // namespace moe
