// Argument block and launcher of the weight-streaming grouped FFN kernel.
#pragma once

#include "common.cuh"

namespace moe {

enum Fmt : int { kBF16 = MOE_W_BF16, kMXFP4 = MOE_W_MXFP4, kNVFP4 = MOE_W_NVFP4, kINT4 = MOE_W_INT4_G128 };

struct FfnArgs {
  // routed experts
  const uint8_t* w;
  const uint8_t* s;
  const float* gsc;
  int64_t stride_w, stride_s;
  const int32_t* slot_map;
  int n_phys;
  // shared experts
  const uint8_t* w_sh;
  const uint8_t* s_sh;
  const float* gsc_sh;
  int64_t stride_w_sh, stride_s_sh;
  int n_shared;
  // problem
  int E, T, k;
  int N;      // output rows of the matrix: d_ff (stage 1: gate rows; up rows follow) or d (stage 2)
  int K;      // reduction length
  const int32_t* offsets;    // [E+1]
  const int32_t* row_token;  // [T*k]
  // B operand source rows (f16 for 4-bit formats, bf16 for BF16), K elements each
  const uint8_t* xsrc;
  const int32_t* xexp;  // per source row power-of-two exponent (4-bit formats)
  // outputs (bf16): routed rows and shared rows
  __nv_bfloat16* out_routed;  // [T*k][N] (stage 1: [rows_total][d_ff] with shared rows after routed)
  __nv_bfloat16* out_shared;  // stage 2: [n_shared][T][N]
  int n_stages;
  int n_scale_buf;
  int smem_scale_bytes;  // per buffer
};

// Launch one stage (gate_up: stage 1 with SwiGLU; else stage 2) of the
// streaming FFN.  Sets *unsupported when the shared-memory plan cannot fit.
cudaError_t launch_ffn_stream(int F, bool gate_up, FfnArgs a, int T, int n_sms, int smem_max, cudaStream_t st,
                              int* unsupported);

}  // namespace moe
