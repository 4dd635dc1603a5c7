// Token permutation into per-expert groups, activation preparation, and the
// weighted combine back to token order.
//
// Grouping: tokens that select the same expert are grouped so that one read of
// the expert's weights serves all of them ("Understanding MoE Inference Costs
// on Galactus", section "Prompt processing is a different phase").  The
// grouping is a stable counting sort of the T*k (token, slot) pairs by expert:
// per-expert counts, their exclusive prefix sum (offsets), then each pair's
// row = offsets[e] + (number of earlier pairs with the same expert).  One
// 1024-thread block does it: shared-memory histogram, block scan, then warp w
// scans the pairs for experts w, w+32, ... with warp ballots, so the result
// is independent of thread scheduling.
//
// Combine: out[t] = sum_j g[t,j] * y[inv[t*k+j]] + sum_s y_shared[s][t], fp32
// in that order ("Each token is sent to the shared expert and also to one of
// the 128 routed experts": "Mixture of experts VRAM: total vs active
// parameters", section "How current MoE models route each token").
#include "common.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "route_device.cuh"

namespace moe {

constexpr int kPermThreads = 1024;
constexpr int kPermTile = 8192;

__global__ void __launch_bounds__(kPermThreads)
    permute_kernel(const int32_t* __restrict__ idx, int n, int k, int E, int32_t* __restrict__ offsets,
                   int32_t* __restrict__ row_token, int32_t* __restrict__ inv) {
  extern __shared__ int sm[];
  int* counts = sm;            // [E]
  int* cursor = sm + E;        // [E]
  int* tile = sm + 2 * E;      // [kPermTile]
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait_and_trigger();
  for (int e = tid; e < E; e += kPermThreads) counts[e] = 0;
  __syncthreads();
  // (a batch that fits one tile keeps its indices in shared memory for the
  // scatter below, which then reads no global memory)
  const bool one_tile = n <= kPermTile;
  for (int i = tid; i < n; i += kPermThreads) {
    const int e = __ldg(idx + i);
    if (one_tile) tile[i] = e;
    if (e < 0 || e >= E) {
      set_status(MOE_ERR_DEVICE_INDEX);
      inv[i] = -1;
    } else {
      atomicAdd(&counts[e], 1);
    }
  }
  __syncthreads();
  // exclusive scan over E <= 1024 counts (one per thread)
  const int v = tid < E ? counts[tid] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    wsum[lane] = wi - w;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - v + wsum[warp];
  if (tid < E) {
    cursor[tid] = excl;
    offsets[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + v;
  }
  __syncthreads();
  for (int base = 0; base < n; base += kPermTile) {
    const int tn = min(kPermTile, n - base);
    if (!one_tile) {
      for (int i = tid; i < tn; i += kPermThreads) tile[i] = __ldg(idx + base + i);
      __syncthreads();
    }
    for (int e = warp; e < E; e += kPermThreads / 32) {
      int run = cursor[e];
      for (int c0 = 0; c0 < tn; c0 += 32) {
        const int i = c0 + lane;
        const bool hit = i < tn && tile[i] == e;
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (hit) {
          const int r = run + __popc(m & ((1u << lane) - 1u));
          row_token[r] = (base + i) / k;
          inv[base + i] = r;
        }
        run += __popc(m);
      }
      if (lane == 0) cursor[e] = run;
    }
    __syncthreads();
  }
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* row_token,
                           int32_t* inv, cudaStream_t st) {
  const size_t smem = (size_t)(2 * E + kPermTile) * sizeof(int);
  cudaError_t err = set_dyn_smem_once<permute_kernel>(smem);
  if (err != cudaSuccess) return err;
  ProfScope prof("permute", st);
  return launch_pdl(permute_kernel, dim3(1), dim3(kPermThreads), smem, st, idx, T * k, k, E, offsets, row_token,
                    inv);
}

// ---------------------------------------------------------------------------
// Activation rows for the grouped FFN, written in expert order so that an
// expert's rows are contiguous.  Output row r reads source row gather[r] for
// r < n_gather and row (r - n_gather) % n_tok after that (the shared experts'
// copies of every token); with no gather array, row r reads row r.
// Modes: kCopyBf16 copies the bf16 row; otherwise the row is converted to fp16
// after scaling by 2^-p with p = floor(log2(max|row|)) - 14, so that its
// largest magnitude lies in [2^14, 2^15) (fp16's range), and rexp[r] = p is
// undone on the accumulators.  kF16Int4 serves the INT4 decode, which meets
// even K with 1024 + (q + 8) and odd K with 1024 + 16 (q + 8): it divides the
// odd-K values by 16 (a power of two), stores each 8-element group in the
// order 0,4,1,5,2,6,3,7 (the decoder's pairing), and writes per 128-wide
// scale group g the constant part of the products,
//   gbias[r][g] = 1032 * sum_{even k in g} h_k + 1152 * sum_{odd k in g} h_k,
// over the stored fp16 values h (summed in fp64, rounded once to fp32), so
// that the grouped FFN recovers sum_k x_k q_k = MMA - gbias exactly up to
// rounding.
// One thread per 8-element chunk of a row (rounded up to whole warps, at
// least 128 and at most 1024): a row's loads are then one round deep.
constexpr int kRowThreadsMin = 128, kRowThreadsMax = 1024;
static int row_threads(int K) {
  int t = ((K / 8 + 31) / 32) * 32;
  return t < kRowThreadsMin ? kRowThreadsMin : (t > kRowThreadsMax ? kRowThreadsMax : t);
}
template <int kMode>
__global__ void __launch_bounds__(kRowThreadsMax)
    prep_rows_kernel(const __nv_bfloat16* __restrict__ src, int K, void* __restrict__ dst,
                     int32_t* __restrict__ rexp, float* __restrict__ gbias, const int32_t* __restrict__ gather,
                     int n_gather, int n_tok, int32_t* __restrict__ zero, int n_zero) {
  pdl_wait_and_trigger();
  __shared__ float red[kRowThreadsMax / 32];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nth = blockDim.x;
  for (int i = row * nth + tid; i < n_zero; i += gridDim.x * nth) zero[i] = 0;
  int srow = row;
  if (gather) srow = row < n_gather ? __ldg(gather + row) : (row - n_gather) % n_tok;
  // a gathered row past the grouped rows (a pair the permutation dropped)
  // has no source: it is written as zeros
  const bool have = !gather || (unsigned)srow < (unsigned)n_tok;
  const __nv_bfloat16* s = have ? src + (size_t)srow * K : nullptr;
  const size_t esz = kMode == kCopyBf16 ? sizeof(__nv_bfloat16) : sizeof(__half);
  void* d = static_cast<uint8_t*>(dst) + (size_t)row * K * esz;
  prep_row<kMode>(s, K, d, rexp ? rexp + row : nullptr, gbias ? gbias + (size_t)row * (K / 128) : nullptr, tid, nth,
                  red);
}

// mode: 0 fp16 scaled, 1 fp16 scaled for the INT4 decode (+ gbias), 2 bf16 copy.
// zero[0..n_zero) is cleared on the way (counters the next kernels start from).
cudaError_t launch_prep_rows(const void* src, int rows, int K, int mode, void* dst, int32_t* rexp, float* gbias,
                             const int32_t* gather, int n_gather, int n_tok, int32_t* zero, int n_zero,
                             cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  ProfScope prof(gather ? "prep_x_gather" : "prep_h", st);
  const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src);
  if (mode == kCopyBf16)
    return launch_pdl(prep_rows_kernel<kCopyBf16>, dim3(rows), dim3(row_threads(K)), 0, st, s, K, dst, rexp, gbias,
                      gather, n_gather, n_tok, zero, n_zero);
  if (mode == kF16Int4)
    return launch_pdl(prep_rows_kernel<kF16Int4>, dim3(rows), dim3(row_threads(K)), 0, st, s, K, dst, rexp, gbias,
                      gather, n_gather, n_tok, zero, n_zero);
  return launch_pdl(prep_rows_kernel<kF16>, dim3(rows), dim3(row_threads(K)), 0, st, s, K, dst, rexp, gbias, gather,
                    n_gather, n_tok, zero, n_zero);
}

// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kRowThreadsMax)
    combine_kernel(const __nv_bfloat16* __restrict__ y, const int32_t* __restrict__ inv,
                   const float* __restrict__ gw, const __nv_bfloat16* __restrict__ y_shared, int n_shared, int T,
                   int d, int k, __nv_bfloat16* __restrict__ out) {
  pdl_wait_and_trigger();
  const int t = blockIdx.x;
  const int nchunk = d / 8;
  const int nrows = T * k;
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int r = __ldg(inv + (size_t)t * k + j);
      if (r < 0 || r >= nrows) {
        set_status(MOE_ERR_DEVICE_INDEX);
        continue;
      }
      const float g = __ldg(gw + (size_t)t * k + j);
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(y + (size_t)r * d) + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = fmaf(g, bf16_bits_to_f32(w[q] & 0xffffu), acc[2 * q]);
        acc[2 * q + 1] = fmaf(g, bf16_bits_to_f32(w[q] >> 16), acc[2 * q + 1]);
      }
    }
    for (int s = 0; s < n_shared; ++s) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(y_shared + ((size_t)s * T + t) * d) + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += bf16_bits_to_f32(w[q] & 0xffffu);
        acc[2 * q + 1] += bf16_bits_to_f32(w[q] >> 16);
      }
    }
    __nv_bfloat16 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = __float2bfloat16_rn(acc[q]);
    reinterpret_cast<uint4*>(out + (size_t)t * d)[c] = *reinterpret_cast<uint4*>(o);
  }
}

cudaError_t launch_combine(const void* y, const int32_t* inv, const float* gw, const void* y_shared, int n_shared,
                           int T, int d, int k, void* out, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  ProfScope prof("combine", st);
  return launch_pdl(combine_kernel, dim3(T), dim3(row_threads(d)), 0, st, static_cast<const __nv_bfloat16*>(y), inv,
                    gw, static_cast<const __nv_bfloat16*>(y_shared), n_shared, T, d, k,
                    static_cast<__nv_bfloat16*>(out));
}

}  // namespace moe
