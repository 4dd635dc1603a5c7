// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (prefill).
//
// Prefill processes many positions together, so the tokens that select one
// expert form a real matrix and one read of the expert's weights serves all of
// them ("Understanding MoE Inference Costs on Galactus", section "Prompt
// processing is a different phase").  Each expert's rows (activation rows in
// expert order) times its weight matrix is a dense GEMM; this kernel runs all
// of them as one persistent grouped GEMM:
//   stage 1: D = X_e [128 x K] * [W_gate rows n0..n0+127 ; W_up rows n0..n0+127]^T,
//            h = silu(D[:, :128]) * D[:, 128:]      (SwiGLU in the epilogue)
//   stage 2: y = H_e [128 x K] * W_down[n0..n0+255]^T
// (gate / up / down projections: FloE verdict page, JSON field
// referee_report.summary).
//
// CTA = 6 warps, one CTA per SM, persistent over 128 x 256 output tiles
// (m fastest inside an expert, so concurrently running CTAs share each weight
// tile through L2):
//   warp 0 (one lane): TMA loads of A (128 rows x 64 K) and B (256 rows x 64 K)
//                      into a 4-stage ring of 128-byte-swizzled shared memory;
//   warp 1 (one lane): tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M=128,
//                      N=256, K=16 per instruction, accumulating in tensor
//                      memory; 2 accumulators of 256 columns so the epilogue
//                      of one tile overlaps the MMAs of the next; warp 1 also
//                      allocates and frees the 512 TMEM columns;
//   warps 2-5        : epilogue, one TMEM lane (= one output row) per thread:
//                      tcgen05.ld, SwiGLU / conversion, bf16 stores.
// Every wait is bounded (2 s); on expiry the CTA records MOE_ERR_TIMEOUT,
// drains its in-flight copies and MMAs, frees its TMEM and exits.
#include <cstdlib>

#include "ffn_gemm_tc.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;             // rows of A (activation rows) per tile
constexpr int kBN = 256;             // rows of B (weight rows) per tile
constexpr int kBK = 64;              // K per stage: 64 bf16 = 128 bytes = one swizzle line
constexpr int kStages = 4;
constexpr int kABytes = kBM * 128;
constexpr int kBBytes = kBN * 128;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreadsTc = 192;
constexpr int kTmemCols = 512;
constexpr int kMaxGroups = 1024 + 64;

struct TileInfo {
  int group;
  int shared_idx;  // >= 0 for a shared expert
  int xrow0;       // first activation row of the group
  int n_cols;      // activation rows of the group
  int phys;        // weight index (TMA coordinate)
  int m_idx, n_idx;
};

}  // namespace

template <bool kGateUp>
__global__ void __launch_bounds__(kThreadsTc, 1) ffn_gemm_tc_kernel(const __grid_constant__ GemmArgs a) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;  // kStages x (A | B)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_ngroups = reinterpret_cast<int*>(s_tmem + 2);
  int* s_gtile = s_ngroups + 2;            // [kMaxGroups + 1] first m-tile of each group (prefix)
  int* s_gexpert = s_gtile + kMaxGroups + 1;  // [kMaxGroups] expert (routed) or -1 - shared index

  const int n_tiles_n = kGateUp ? a.N / 128 : a.N / kBN;
  const int ksteps = a.K / kBK;
  const int E = a.E;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  pdl_wait_and_trigger();
  // Group table: shared experts first, then routed experts with rows, each
  // with its number of 128-row m-tiles (non-resident experts get none).
  if (warp == 0) {
    int ng = 0, tiles = 0;
    for (int s = 0; s < a.n_shared; ++s) {
      if (lane == 0) {
        s_gtile[ng] = tiles;
        s_gexpert[ng] = -1 - s;
      }
      ++ng;
      tiles += ceil_div(a.T, kBM);
    }
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int mt = 0;
      if (e < E) {
        const int cnt = __ldg(a.offsets + e + 1) - __ldg(a.offsets + e);
        int p = a.slot_map ? __ldg(a.slot_map + e) : e;
        bool ok = cnt > 0;
        if (ok && (p < 0 || p >= a.n_phys)) {
          if (!(p == -1 && a.slot_map)) set_status(MOE_ERR_DEVICE_INDEX);
          ok = false;
        }
        mt = ok ? ceil_div(cnt, kBM) : 0;
      }
      const uint32_t on = __ballot_sync(0xffffffffu, mt > 0);
      int incl = mt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (mt > 0) {
        const int slot = ng + __popc(on & ((1u << lane) - 1u));
        s_gtile[slot] = tiles + incl - mt;
        s_gexpert[slot] = e;
      }
      ng += __popc(on);
      tiles += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_gtile[ng] = tiles;
      *s_ngroups = ng;
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(s_tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const int ngroups = *s_ngroups;
  const int total_tiles = s_gtile[ngroups] * n_tiles_n;

  auto decode = [&](int t) {
    TileInfo ti;
    // groups are laid out as [m_tiles_g x n_tiles] blocks; binary search on the scaled prefix
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_gtile[mid] * n_tiles_n <= t) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int mtg = s_gtile[g + 1] - s_gtile[g];
    const int local = t - s_gtile[g] * n_tiles_n;
    ti.group = g;
    ti.n_idx = local / mtg;
    ti.m_idx = local - ti.n_idx * mtg;
    const int ex = s_gexpert[g];
    if (ex < 0) {
      ti.shared_idx = -1 - ex;
      ti.xrow0 = a.T * a.k + ti.shared_idx * a.T;
      ti.n_cols = a.T;
      ti.phys = ti.shared_idx;
    } else {
      ti.shared_idx = -1;
      ti.xrow0 = __ldg(a.offsets + ex);
      ti.n_cols = __ldg(a.offsets + ex + 1) - ti.xrow0;
      ti.phys = a.slot_map ? __ldg(a.slot_map + ex) : ex;
    }
    return ti;
  };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      prefetch_tmap(&a.tm_a);
      prefetch_tmap(&a.tm_b);
      if (a.n_shared) prefetch_tmap(&a.tm_bsh);
      const uint64_t pol_b = l2_evict_last_policy();  // weight tiles are re-read by the other m-tiles
      const uint64_t pol_a = l2_evict_last_policy();
      uint32_t cnt = 0;
      for (int t = blockIdx.x; t < total_tiles && !*s_abort; t += gridDim.x) {
        const TileInfo ti = decode(t);
        const CUtensorMap* tb = ti.shared_idx >= 0 ? &a.tm_bsh : &a.tm_b;
        const int arow = ti.xrow0 + ti.m_idx * kBM;
        const int n0 = ti.n_idx * (kGateUp ? 128 : kBN);
        for (int ks = 0; ks < ksteps; ++ks) {
          const int s = cnt % kStages;
          if (!mbar_wait(&empty[s], ((cnt / kStages) & 1u) ^ 1u)) {
            *s_abort = 1;
            break;
          }
          uint8_t* sa = stages + s * kStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(sa, &a.tm_a, ks * 128, arow, &full[s], pol_a);
          if (kGateUp) {
            tma_load_3d(sb, tb, ks * 128, n0, ti.phys, &full[s], pol_b);
            tma_load_3d(sb + 128 * 128, tb, ks * 128, a.N + n0, ti.phys, &full[s], pol_b);
          } else {
            tma_load_3d(sb, tb, ks * 128, n0, ti.phys, &full[s], pol_b);
            tma_load_3d(sb + 128 * 128, tb, ks * 128, n0 + 128, ti.phys, &full[s], pol_b);
          }
          ++cnt;
        }
      }
      const uint32_t first = cnt > (uint32_t)kStages ? cnt - kStages : 0;
      for (uint32_t c = first; c < cnt; ++c) mbar_wait(&full[c % kStages], (c / kStages) & 1u);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kBM, kBN);
      uint32_t cnt = 0;
      int i = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < total_tiles && !*s_abort; t += gridDim.x, ++i) {
        const int buf = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u)) {
          *s_abort = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * kBN);
        for (int ks = 0; ks < ksteps; ++ks) {
          const int s = cnt % kStages;
          if (!mbar_wait(&full[s], (cnt / kStages) & 1u)) {
            *s_abort = 1;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa = smem_u32(stages + s * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc::mma_bf16(d_tmem, tc::kmajor_sw128_desc(sa + kk * 32), tc::kmajor_sw128_desc(sb + kk * 32), idesc,
                         (ks | kk) != 0 ? 1u : 0u);
          tc::commit(&empty[s]);  // frees the stage once these MMAs have read it
          issued = true;
          ++cnt;
        }
        if (*s_abort) break;
        tc::commit(&acc_full[buf]);
      }
      if (issued) {  // every MMA of this CTA has completed before TMEM is freed
        tc::commit(drain);
        mbar_wait(drain, 0);
      }
    }
  } else {
    // ================================================================ epilogue
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;
    int i = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++i) {
      const int buf = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      if (*s_abort || !mbar_wait(&acc_full[buf], use & 1u)) {
        *s_abort = 1;
        break;
      }
      tc::fence_after_sync();
      const TileInfo ti = decode(t);
      const int m = ti.m_idx * kBM + r;  // row inside the group
      const bool valid = m < ti.n_cols;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kBN);
      if (kGateUp) {
        __nv_bfloat16* o = a.out_routed + (int64_t)(ti.xrow0 + m) * a.N + ti.n_idx * 128;
#pragma unroll 1
        for (int j0 = 0; j0 < 128; j0 += 32) {
          uint32_t gv[32], uv[32];
          tc::ld_32x32b_x32(taddr + j0, gv);
          tc::ld_32x32b_x32(taddr + 128 + j0, uv);
          tc::ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(gv[2 * j]), g1 = __uint_as_float(gv[2 * j + 1]);
              const float u0 = __uint_as_float(uv[2 * j]), u1 = __uint_as_float(uv[2 * j + 1]);
              const float h0 = g0 / (1.f + __expf(-g0)) * u0;
              const float h1 = g1 / (1.f + __expf(-g1)) * u1;
              __nv_bfloat162 hb = __floats2bfloat162_rn(h0, h1);
              packed[j] = *reinterpret_cast<uint32_t*>(&hb);
            }
            uint4* dst = reinterpret_cast<uint4*>(o + j0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
      } else {
        __nv_bfloat16* o = ti.shared_idx >= 0 ? a.out_shared + ((int64_t)ti.shared_idx * a.T + m) * a.N
                                              : a.out_routed + (int64_t)(ti.xrow0 + m) * a.N;
        o += ti.n_idx * kBN;
#pragma unroll 1
        for (int j0 = 0; j0 < kBN; j0 += 32) {
          uint32_t v[32];
          tc::ld_32x32b_x32(taddr + j0, v);
          tc::ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
              packed[j] = *reinterpret_cast<uint32_t*>(&hb);
            }
            uint4* dst = reinterpret_cast<uint4*>(o + j0);
#pragma unroll
            for (int w = 0; w < 4; ++w)
              dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1], packed[4 * w + 2], packed[4 * w + 3]);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------ host side
bool gemm_path_supported(int F, int N, int K, bool gate_up) {
  if (F != MOE_W_BF16) return false;
  if (K % kBK) return false;
  return gate_up ? (N % 128 == 0) : (N % kBN == 0);
}

template <bool GU>
static cudaError_t launch_gemm(const GemmArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto kern = ffn_gemm_tc_kernel<GU>;
  {
    cudaError_t err = set_dyn_smem_once<ffn_gemm_tc_kernel<GU>>(smem);
    if (err != cudaSuccess) return err;
  }
  ProfScope prof(GU ? "ffn_gemm_stage1_gate_up" : "ffn_gemm_stage2_down", st);
  return launch_pdl(kern, dim3(grid), dim3(kThreadsTc), smem, st, a);
}

cudaError_t launch_ffn_gemm(bool gate_up, GemmArgs a, const GemmPointers& p, int n_sms, int smem_max,
                            cudaStream_t st, int* unsupported) {
  *unsupported = 0;
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + 1024 + (size_t)(2 * kMaxGroups + 8) * 4;
  if ((int)smem > smem_max || !gemm_path_supported(MOE_W_BF16, a.N, a.K, gate_up)) {
    *unsupported = 1;
    return cudaSuccess;
  }
  const uint64_t row_bytes = (uint64_t)a.K * 2;
  const uint64_t wrows = gate_up ? 2 * (uint64_t)a.N : (uint64_t)a.N;
  {
    const uint64_t dims[2] = {row_bytes, (uint64_t)p.rows_total};
    const uint64_t strides[1] = {row_bytes};
    const uint32_t box[2] = {128, kBM};
    if (!encode_tmap_u8(&a.tm_a, p.x, 2, dims, strides, box, true)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  }
  {
    const uint64_t dims[3] = {row_bytes, wrows, (uint64_t)a.n_phys};
    const uint64_t strides[2] = {row_bytes, (uint64_t)p.stride_w};
    const uint32_t box[3] = {128, 128, 1};
    if (!encode_tmap_u8(&a.tm_b, p.w, 3, dims, strides, box, true)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  }
  if (a.n_shared > 0) {
    const uint64_t dims[3] = {row_bytes, wrows, (uint64_t)a.n_shared};
    const uint64_t strides[2] = {row_bytes, (uint64_t)p.stride_w_sh};
    const uint32_t box[3] = {128, 128, 1};
    if (!encode_tmap_u8(&a.tm_bsh, p.w_sh, 3, dims, strides, box, true)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  } else {
    a.tm_bsh = a.tm_b;
  }
  const int n_tiles_n = gate_up ? a.N / 128 : a.N / kBN;
  const long rows = (long)a.T * a.k;
  const long max_mtiles = (rows + kBM - 1) / kBM + (a.E < rows ? a.E : rows) + (long)a.n_shared * ((a.T + kBM - 1) / kBM);
  const long max_tiles = max_mtiles * n_tiles_n;
  const int grid = (int)(max_tiles < n_sms ? max_tiles : n_sms);
  if (grid < 1) return cudaSuccess;
  return gate_up ? launch_gemm<true>(a, grid, smem, st) : launch_gemm<false>(a, grid, smem, st);
}

}  // namespace moe
