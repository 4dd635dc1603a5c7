// C ABI entry points of the MoE layer library: argument checks, workspace
// layout, and the order in which the kernels of one layer are enqueued.
//
// One layer call (page "Mixture of experts VRAM: total vs active parameters",
// section "How current MoE models route each token": a router picks a few
// experts per token; Galactus page, section "Prompt processing is a different
// phase": tokens of one expert are grouped) runs, on the caller's stream:
//   router logits -> top-k + gates -> stable permutation ->
//   [4-bit: activation rows to fp16] -> stage 1 (gate/up + SwiGLU) ->
//   [4-bit: h rows to fp16] -> stage 2 (down) -> weighted combine.
// Nothing here allocates device memory; all scratch is carved from the
// caller's workspace.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ffn_gemm_tc.cuh"

namespace moe {

__device__ int g_status = 0;

cudaError_t launch_route_topk(const moe_layer_desc& dsc, const void* x, const void* wr, const float* bias,
                              float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st);
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* row_token,
                           int32_t* inv, cudaStream_t st);
cudaError_t launch_prep_rows(const void* src, int rows, int K, int mode, void* dst, int32_t* rexp, float* gbias,
                             const int32_t* gather, int n_gather, int n_tok, int32_t* zero, int n_zero,
                             cudaStream_t st);
cudaError_t launch_combine(const void* y, const int32_t* inv, const float* gw, const void* y_shared, int n_shared,
                           int T, int d, int k, void* out, cudaStream_t st);
bool route_prep_small_supported(const moe_layer_desc& d);
cudaError_t launch_route_prep_small(const moe_layer_desc& dsc, const void* x, const void* wr, const float* bias,
                                    int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* row_token,
                                    int32_t* inv, int mode, void* xperm, int32_t* xexp, float* gbias, int32_t* zero,
                                    int n_zero, cudaStream_t st);

}  // namespace moe

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int fmt_block(int f) {
  switch (f) {
    case MOE_W_MXFP4: return 32;
    case MOE_W_NVFP4: return 16;
    case MOE_W_INT4_G128: return 128;
    default: return 1;
  }
}
int fmt_scale_bytes(int f) { return f == MOE_W_INT4_G128 ? 2 : (f == MOE_W_BF16 ? 0 : 1); }
bool is4bit(int f) { return f != MOE_W_BF16; }

// bytes of one [N][K] matrix's values / scales
int64_t mat_bytes(int f, int64_t N, int64_t K) { return is4bit(f) ? N * K / 2 : N * K * 2; }
int64_t scale_bytes(int f, int64_t N, int64_t K) {
  return is4bit(f) ? N * (K / fmt_block(f)) * fmt_scale_bytes(f) : 0;
}

struct Layout {
  size_t logits, topk_idx, topk_w, offsets, row_token, inv, xperm, xexp, gbias, h, hq, hexp, y, ysh, ctr, split_part,
      total;
  int n_ctr;  // int32 counters at ctr, zeroed by the activation-prep kernel of every call
};

// Batches of at most this many tokens may split the streaming FFN's items
// along K (MOE_FFN_SPLIT=S, off by default); their workspace holds the split
// counters and partial sums.
constexpr int kSplitMaxT = 8;

// Counters the activation-prep kernel zeroes: the two work counters, plus the
// split-K arrival counters when a split is asked for.
int counters_to_zero(const Layout& L) {
  if (L.n_ctr <= 2) return 2;
  const char* e = std::getenv("MOE_FFN_SPLIT");
  return (e && std::atoi(e) > 1) ? L.n_ctr : 2;
}

Layout layout_of(const moe_layer_desc& d) {
  Layout L{};
  const size_t T = d.T, E = d.n_experts, k = d.top_k, D = d.d_model, F = d.d_ff, S = d.n_shared;
  const size_t R = T * k, RT = R + S * T;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.logits = take(T * E * 4);
  L.topk_idx = take(T * k * 4);
  L.topk_w = take(T * k * 4);
  L.offsets = take((E + 1) * 4);
  L.row_token = take(R * 4);
  L.inv = take(R * 4);
  const bool q = is4bit(d.wdtype);
  L.xperm = take(RT * D * 2);
  L.xexp = take(q ? RT * 4 : 0);
  // INT4: per row and 128-wide scale group, stage 1 (K = d) then reused by stage 2 (K = d_ff)
  L.gbias = take(d.wdtype == MOE_W_INT4_G128 ? RT * ((D > F ? D : F) / 128) * 4 : 0);
  L.h = take(RT * F * 2);
  L.hq = take(q ? RT * F * 2 : 0);
  L.hexp = take(q ? RT * 4 : 0);
  L.y = take(R * D * 2);
  L.ysh = take(S * T * D * 2);
  // work counters of the two streaming FFN stages, then (small batches) each
  // stage's split-K arrival counters
  const bool split = d.T <= kSplitMaxT;
  L.n_ctr = 2 + (split ? 2 * kStreamSplitCtrInts : 0);
  L.ctr = take((size_t)L.n_ctr * 4);
  L.split_part = take(split ? kStreamSplitPartBytes : 0);  // shared by both stages (they run in turn)
  L.total = o;
  return L;
}

moe_status check_desc(const moe_layer_desc* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->d_model <= 0 || d->d_ff <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->n_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (d->wdtype < MOE_W_BF16 || d->wdtype > MOE_W_INT4_G128) return MOE_ERR_INVALID_ARG;
  if (d->router_fp32 != 0 && d->router_fp32 != 1) return MOE_ERR_INVALID_ARG;
  const int blk = d->wdtype == MOE_W_INT4_G128 ? 128 : 32;
  if (d->d_model % blk || d->d_ff % blk) return MOE_ERR_INVALID_ARG;
  if (d->top_k > d->n_experts || d->top_k > 32) return MOE_ERR_INVALID_ARG;
  if (d->n_experts > 1024 || d->n_shared > 64) return MOE_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)d->T * d->top_k + (int64_t)d->n_shared * d->T;
  if (rows * (int64_t)(d->d_ff > d->d_model ? d->d_ff : d->d_model) > (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct DevInfo {
  int sms = 0, smem_optin = 0, smem_per_sm = 0;
};

DevInfo dev_info() {
  static std::mutex mu;
  static DevInfo cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev].sms == 0) {
    cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&cache[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&cache[dev].smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  }
  return cache[dev];
}

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Fill the stream-kernel arguments of one stage.
moe_status check_weights(const moe_layer_desc& d, const moe_weights* w, int n_expected) {
  if (!w || !w->w13 || !w->w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w13) || !aligned16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (is4bit(d.wdtype)) {
    if (!w->s13 || !w->s2 || !aligned16(w->s13) || !aligned16(w->s2)) return MOE_ERR_INVALID_ARG;
  }
  if (d.wdtype == MOE_W_NVFP4 && (!w->g13 || !w->g2)) return MOE_ERR_INVALID_ARG;
  if ((w->stride_w13 | w->stride_s13 | w->stride_w2 | w->stride_s2) & 15) return MOE_ERR_INVALID_ARG;
  if (w->stride_w13 < 0 || w->stride_s13 < 0 || w->stride_w2 < 0 || w->stride_s2 < 0) return MOE_ERR_INVALID_ARG;
  if (w->n_physical < 0) return MOE_ERR_INVALID_ARG;
  (void)n_expected;
  return MOE_OK;
}

// Which FFN path a call takes, and the activation-row format that path reads.
struct FfnPlan {
  bool use_gemm;     // tensor-core grouped GEMM (else the weight-streaming kernel)
  bool q_bf16_acts;  // 4-bit on the GEMM path with bf16 activation rows (MXFP4)
  bool int4_stream;  // INT4 on the streaming path (offset decode: reordered rows + group constants)
  int mode;          // activation prep: 0 fp16 scaled, 1 fp16 scaled for the INT4 decode, 2 bf16 copy
};

FfnPlan ffn_plan(const moe_layer_desc& d) {
  const int f = d.wdtype;
  const bool q = is4bit(f);
  const int F = d.d_ff, D = d.d_model;
  // Path: the tcgen05 grouped GEMM when experts average at least 64 rows
  // (prefill-sized groups; bf16 weights, or 4-bit weights decoded to 16-bit
  // tiles in shared memory), else the weight-streaming kernel.
  // MOE_FFN_PATH=stream|gemm overrides the choice where both can run.
  const bool gemm_ok = q ? (gemm_q4_supported(f, F, D, true) && gemm_q4_supported(f, D, F, false))
                         : (gemm_path_supported(f, F, D, true) && gemm_path_supported(f, D, F, false));
  FfnPlan p{};
  p.use_gemm = gemm_ok && (int64_t)d.T * d.top_k >= 64LL * d.n_experts;
  if (const char* e = getenv("MOE_FFN_PATH")) {
    if (!strcmp(e, "stream")) p.use_gemm = false;
    if (!strcmp(e, "gemm")) p.use_gemm = gemm_ok;
  }
  // Activation rows: bf16 copies (bf16 weights; MXFP4 on the tensor-core
  // path), fp16 scaled by a power of two per row (the 4-bit formats
  // otherwise), for the streaming INT4 decode also reordered with the
  // per-group constants.
  p.q_bf16_acts = q && p.use_gemm && gemm_q4_bf16_activations(f);
  p.int4_stream = f == MOE_W_INT4_G128 && !p.use_gemm;
  p.mode = (!q || p.q_bf16_acts) ? 2 : (p.int4_stream ? 1 : 0);
  return p;
}

// x_prepped: the activation rows (and the stage counters) were already
// written by the fused small-batch routing kernel.
moe_status grouped_ffn_impl(const moe_layer_desc& d, const moe_weights* routed, const moe_weights* shared,
                            const int32_t* offsets, const int32_t* row_token, const void* x, void* y_perm,
                            void* y_shared, uint8_t* ws, cudaStream_t st, bool x_prepped = false) {
  const Layout L = layout_of(d);
  const int f = d.wdtype;
  const bool q = is4bit(f);
  const int T = d.T, D = d.d_model, F = d.d_ff, S = d.n_shared, E = d.n_experts, k = d.top_k;
  const int R = T * k, RT = R + S * T;
  const DevInfo di = dev_info();
  cudaError_t err;
  void* xperm = ws + L.xperm;
  int32_t* xexp = reinterpret_cast<int32_t*>(ws + L.xexp);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  __half* hq = reinterpret_cast<__half*>(ws + L.hq);
  int32_t* hexp = reinterpret_cast<int32_t*>(ws + L.hexp);
  const FfnPlan plan = ffn_plan(d);
  const bool use_gemm = plan.use_gemm, q_bf16_acts = plan.q_bf16_acts;
  float* gbias = plan.int4_stream ? reinterpret_cast<float*>(ws + L.gbias) : nullptr;
  const int mode = plan.mode;
  // activation rows in expert order (routed rows, then every token once per shared expert)
  // (also zeroes the work counters of both FFN stages)
  int32_t* ctr = reinterpret_cast<int32_t*>(ws + L.ctr);
  if (!x_prepped) {
    err = launch_prep_rows(x, RT, D, mode, xperm, xexp, gbias, row_token, R, T, ctr, counters_to_zero(L), st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  auto fill = [&](FfnArgs& a, FfnPointers& p, bool stage1) {
    std::memset(&a, 0, sizeof(a));
    std::memset(&p, 0, sizeof(p));
    const int64_t N = stage1 ? 2 * (int64_t)F : D, K = stage1 ? D : F;
    const int64_t sw = stage1 ? routed->stride_w13 : routed->stride_w2;
    const int64_t ss = stage1 ? routed->stride_s13 : routed->stride_s2;
    p.w = stage1 ? routed->w13 : routed->w2;
    p.stride_w = sw ? sw : mat_bytes(f, N, K);
    a.s = static_cast<const uint8_t*>(stage1 ? routed->s13 : routed->s2);
    a.stride_s = ss ? ss : scale_bytes(f, N, K);
    a.gsc = stage1 ? routed->g13 : routed->g2;
    a.slot_map = routed->slot_map;
    a.n_phys = routed->n_physical ? routed->n_physical : E;
    if (S > 0) {
      const int64_t shw = stage1 ? shared->stride_w13 : shared->stride_w2;
      const int64_t shs = stage1 ? shared->stride_s13 : shared->stride_s2;
      p.w_sh = stage1 ? shared->w13 : shared->w2;
      p.stride_w_sh = shw ? shw : mat_bytes(f, N, K);
      a.s_sh = static_cast<const uint8_t*>(stage1 ? shared->s13 : shared->s2);
      a.stride_s_sh = shs ? shs : scale_bytes(f, N, K);
      a.gsc_sh = stage1 ? shared->g13 : shared->g2;
    }
    p.rows_total = RT;
    a.n_shared = S;
    a.E = E;
    a.T = T;
    a.k = k;
    a.N = stage1 ? F : D;
    a.K = (int)K;
    a.offsets = offsets;
  };
  auto to_gemm = [&](const FfnArgs& s) {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    g.offsets = s.offsets;
    g.slot_map = s.slot_map;
    g.n_phys = s.n_phys;
    g.n_shared = s.n_shared;
    g.E = s.E;
    g.T = s.T;
    g.k = s.k;
    g.N = s.N;
    g.K = s.K;
    g.out_routed = s.out_routed;
    g.out_shared = s.out_shared;
    return g;
  };
  // the 4-bit tensor-core stages: argument block and pointers
  auto to_q4 = [&](const FfnArgs& s, const FfnPointers& p, bool stage1, GemmQ4Pointers& qp) {
    GemmQ4Args g;
    std::memset(&g, 0, sizeof(g));
    std::memset(&qp, 0, sizeof(qp));
    g.offsets = s.offsets;
    g.slot_map = s.slot_map;
    g.n_phys = s.n_phys;
    g.n_shared = s.n_shared;
    g.E = s.E;
    g.T = s.T;
    g.k = s.k;
    g.N = s.N;
    g.K = s.K;
    g.gsc = s.gsc;
    g.gsc_sh = s.gsc_sh;
    g.xexp = q_bf16_acts ? nullptr : s.xexp;
    g.out_routed = s.out_routed;
    g.out_shared = s.out_shared;
    qp.w = p.w;
    qp.stride_w = p.stride_w;
    qp.s = s.s;
    qp.stride_s = s.stride_s;
    qp.w_sh = p.w_sh;
    qp.stride_w_sh = p.stride_w_sh;
    qp.s_sh = s.s_sh;
    qp.stride_s_sh = s.stride_s_sh;
    qp.x = p.x;
    qp.rows_total = p.rows_total;
    (void)stage1;
    return g;
  };
  FfnArgs a1;
  FfnPointers p1;
  fill(a1, p1, true);
  p1.x = xperm;
  a1.xexp = q ? xexp : nullptr;
  a1.xbias = gbias;
  a1.work_ctr = ctr;
  const bool split_buffers = counters_to_zero(L) > 2;
  if (split_buffers) {
    a1.split_cap = kStreamSplitCap;
    a1.split_ctr = ctr + 2;
    a1.split_part = reinterpret_cast<float*>(ws + L.split_part);
  }
  a1.out_routed = h;
  a1.out_shared = nullptr;
  int unsup = 0;
  GemmQ4Pointers qp;
  if (use_gemm && q)
    err = launch_ffn_gemm_q4(f, true, to_q4(a1, p1, true, qp), qp, di.sms, di.smem_optin, st, &unsup);
  else if (use_gemm)
    err = launch_ffn_gemm(true, to_gemm(a1), p1, di.sms, di.smem_optin, st, &unsup);
  else
    err = launch_ffn_stream(f, true, a1, p1, T, di.sms, di.smem_optin, di.smem_per_sm, st, &unsup);
  if (unsup) return MOE_ERR_UNSUPPORTED;
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  // h rows for stage 2: as written (bf16) for bf16 operands, else fp16 scaled
  const bool h_f16 = q && !q_bf16_acts;
  if (h_f16) {
    err = launch_prep_rows(h, RT, F, mode, hq, hexp, gbias, nullptr, 0, T, nullptr, 0, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  FfnArgs a2;
  FfnPointers p2;
  fill(a2, p2, false);
  p2.x = h_f16 ? static_cast<const void*>(hq) : static_cast<const void*>(h);
  a2.xexp = h_f16 ? hexp : nullptr;
  a2.xbias = gbias;
  a2.work_ctr = ctr + 1;
  if (split_buffers) {
    a2.split_cap = kStreamSplitCap;
    a2.split_ctr = ctr + 2 + kStreamSplitCtrInts;
    a2.split_part = reinterpret_cast<float*>(ws + L.split_part);
  }
  a2.out_routed = static_cast<__nv_bfloat16*>(y_perm);
  a2.out_shared = static_cast<__nv_bfloat16*>(y_shared);
  if (use_gemm && q)
    err = launch_ffn_gemm_q4(f, false, to_q4(a2, p2, false, qp), qp, di.sms, di.smem_optin, st, &unsup);
  else if (use_gemm)
    err = launch_ffn_gemm(false, to_gemm(a2), p2, di.sms, di.smem_optin, st, &unsup);
  else
    err = launch_ffn_stream(f, false, a2, p2, T, di.sms, di.smem_optin, di.smem_per_sm, st, &unsup);
  if (unsup) return MOE_ERR_UNSUPPORTED;
  return from_cuda(err);
}

}  // namespace

extern "C" {

moe_status moe_workspace_size(const moe_layer_desc* desc, size_t* bytes) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = layout_of(*desc).total;
  return MOE_OK;
}

moe_status moe_workspace_layout_of(const moe_layer_desc* desc, moe_workspace_layout* out) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (!out) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*desc);
  out->topk_idx = L.topk_idx;
  out->topk_w = L.topk_w;
  out->offsets = L.offsets;
  out->row_token = L.row_token;
  out->inv = L.inv;
  out->total = L.total;
  return MOE_OK;
}

moe_status moe_route_topk(const moe_layer_desc* desc, const void* x, const void* w_router, const float* logit_bias,
                          int32_t* topk_idx, float* topk_w, void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (desc->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*desc);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  float* logits = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + L.logits);
  return from_cuda(launch_route_topk(*desc, x, w_router, logit_bias, logits, topk_idx, topk_w,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_layer_desc* desc, const int32_t* topk_idx, const void* x, int32_t* offsets,
                       int32_t* row_token, int32_t* inv, void* x_perm, void* stream) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (desc->T > 0 && (!topk_idx || !row_token || !inv)) return MOE_ERR_INVALID_ARG;
  if (x && desc->T > 0 && (!x_perm || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err = launch_permute(topk_idx, desc->T, desc->top_k, desc->n_experts, offsets, row_token, inv, st);
  if (err != cudaSuccess || !x || desc->T == 0) return from_cuda(err);
  // x_perm[r] = x[row_token[r]] (bf16 rows in expert order)
  const int R = desc->T * desc->top_k;
  return from_cuda(launch_prep_rows(x, R, desc->d_model, 2, x_perm, nullptr, nullptr, row_token, R, desc->T,
                                    nullptr, 0, st));
}

moe_status moe_grouped_ffn(const moe_layer_desc* desc, const moe_weights* routed, const moe_weights* shared,
                           const int32_t* offsets, const int32_t* row_token, const void* x, void* y_perm,
                           void* y_shared, void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (desc->T == 0) return MOE_OK;
  if ((s = check_weights(*desc, routed, desc->n_experts)) != MOE_OK) return s;
  if (desc->n_shared > 0) {
    if ((s = check_weights(*desc, shared, desc->n_shared)) != MOE_OK) return s;
    if (!y_shared || !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
  }
  if (!offsets || !row_token || !x || !y_perm || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y_perm) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < layout_of(*desc).total) return MOE_ERR_WORKSPACE;
  return grouped_ffn_impl(*desc, routed, shared, offsets, row_token, x, y_perm, y_shared,
                          static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

moe_status moe_combine(const moe_layer_desc* desc, const void* y_perm, const int32_t* inv, const float* topk_w,
                       const void* y_shared, void* out, void* stream) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (desc->T == 0) return MOE_OK;
  if (!y_perm || !inv || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (desc->n_shared > 0 && !y_shared) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(out) || (y_shared && !aligned16(y_shared))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_combine(y_perm, inv, topk_w, y_shared, desc->n_shared, desc->T, desc->d_model,
                                  desc->top_k, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(const moe_layer_desc* desc, const void* x, const void* w_router,
                             const float* logit_bias, const moe_weights* routed, const moe_weights* shared,
                             void* out, void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_desc(desc);
  if (s != MOE_OK) return s;
  if (desc->T == 0) return MOE_OK;
  if ((s = check_weights(*desc, routed, desc->n_experts)) != MOE_OK) return s;
  if (desc->n_shared > 0 && (s = check_weights(*desc, shared, desc->n_shared)) != MOE_OK) return s;
  if (!x || !w_router || !out || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(out) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*desc);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  float* gw = reinterpret_cast<float*>(ws + L.topk_w);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* rtok = reinterpret_cast<int32_t*>(ws + L.row_token);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
  const bool fused = route_prep_small_supported(*desc);
  cudaError_t err;
  if (fused) {
    // small batch: router, top-k, permutation and activation rows in one launch
    const FfnPlan plan = ffn_plan(*desc);
    err = launch_route_prep_small(*desc, x, w_router, logit_bias, idx, gw, offs, rtok, inv, plan.mode, ws + L.xperm,
                                  reinterpret_cast<int32_t*>(ws + L.xexp),
                                  plan.int4_stream ? reinterpret_cast<float*>(ws + L.gbias) : nullptr,
                                  reinterpret_cast<int32_t*>(ws + L.ctr), counters_to_zero(L), st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    err = launch_route_topk(*desc, x, w_router, logit_bias, reinterpret_cast<float*>(ws + L.logits), idx, gw, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    err = launch_permute(idx, desc->T, desc->top_k, desc->n_experts, offs, rtok, inv, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  void* y = ws + L.y;
  void* ysh = desc->n_shared ? ws + L.ysh : nullptr;
  s = grouped_ffn_impl(*desc, routed, shared, offs, rtok, x, y, ysh, ws, st, fused);
  if (s != MOE_OK) return s;
  return from_cuda(launch_combine(y, inv, gw, ysh, desc->n_shared, desc->T, desc->d_model, desc->top_k, out, st));
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_OOM: return "out of memory";
    case MOE_ERR_CACHE_PINNED_FULL: return "every cache slot of the layer is protected";
    case MOE_ERR_TIMEOUT: return "a device-side wait timed out";
    case MOE_ERR_INJECTED: return "injected fault";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_DEVICE_INDEX: return "a kernel saw an index out of range";
  }
  return "unknown status";
}

moe_status moe_get_last_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, moe::g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(moe::g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Diagnostic: the bounded wait every pipelined kernel uses, made to run out.
// One CTA waits on an mbarrier phase that nothing completes, with the given
// limit; the wait gives up, records MOE_ERR_TIMEOUT in the status word and
// the kernel returns normally, so the context stays usable.
namespace moe {
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns, int* finished) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_limit(&bar, 0, limit_ns);  // phase 0 never completes
    *finished = ok ? 2 : 1;
  }
}
}  // namespace moe

extern "C" moe_status moe_diag_wait_timeout(uint64_t limit_ns, int32_t* finished, void* stream) {
  if (!finished || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  moe::wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, finished);
  return from_cuda(cudaGetLastError());
}
