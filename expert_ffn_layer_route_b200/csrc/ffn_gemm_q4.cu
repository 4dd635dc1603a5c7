// Grouped SwiGLU expert FFN on the 5th-generation tensor cores for 4-bit
// expert weights (prefill-sized groups).
//
// Prefill groups the tokens that chose one expert so that one read of its
// weights serves all of them ("Understanding MoE Inference Costs on
// Galactus", section "Prompt processing is a different phase"); the 4-bit
// experts are the FP4 and INT4 ones current models ship ("Mixture of experts
// VRAM: total vs active parameters", section "How current MoE models route
// each token").  Per expert the work is a dense GEMM against 4-bit weights:
// the weights are decoded once per tile into 16-bit values in shared memory
// and fed to tcgen05.mma kind::f16, with fp32 accumulation in tensor memory.
//
//   stage 1: D = X_e [256 x K] * [W_gate rows n0..n0+127 ; W_up rows n0..n0+127]^T,
//            h = silu(D[:, :128]) * D[:, 128:]
//   stage 2: y = H_e [256 x K] * W_down[n0..n0+255]^T
//
// Operand types, chosen so that every decoded weight is exact:
//   MXFP4: E2M1 x 2^(s-127) in bf16 (2 significant bits, bf16's exponent
//          range) against the bf16 activation rows;
//   NVFP4: E2M1 x E4M3 in fp16 (at most 6 significant bits, magnitudes in
//          [2^-10, 2688], inside fp16's normal range) against fp16 activation
//          rows scaled by a power of two per row; the per-expert fp32 global
//          scale and the row's power of two are applied to the fp32 result;
//   INT4 : q x s in fp16 (q in [-8, 7], s a bf16 group scale: at most 11
//          significant bits, exact for s in [2^-17, 2^13)) against the same
//          scaled fp16 activation rows.
//
// CTA = 14 warps, one CTA per SM, persistent over tiles of (expert, 256
// activation rows, 256 weight rows); activation rows fastest inside an expert
// so that CTAs running side by side share each weight tile through L2:
//   warp 0 (one lane): TMA loads per 64-wide K step into a 3-stage ring: the
//                      two 128-row activation boxes (128-byte swizzle), the
//                      256 weight rows' codes (32 bytes each) and their
//                      16-byte block-scale segments;
//   warps 6-13       : converters, one weight row per thread: decode the
//                      row's 64 codes with its scales into 128 bytes of
//                      16-bit values (NVFP4 and INT4 by byte-permute table
//                      lookups and 16-bit multiplies, MXFP4 through the
//                      hardware E2M1 conversion: the fastest measured for
//                      each), written in the 128-byte-swizzled K-major
//                      layout the MMA reads, into a 2-slot ring;
//   warp 1 (one lane): tcgen05.mma (M=128, N=256, K=16), one per 128-row
//                      activation half, into 2 x 256 TMEM columns; warp 1
//                      also allocates and frees the 512 columns;
//   warps 2-5        : epilogue, one TMEM lane (= activation row) per thread:
//                      tcgen05.ld, scale, SwiGLU / conversion, bf16 stores.
// Every wait is bounded (2 s); on expiry the CTA records MOE_ERR_TIMEOUT,
// lets its in-flight copies and MMAs land, frees its TMEM and exits.
#include <cstdlib>

#include "ffn_gemm_tc.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

constexpr int kQBM = 128;                 // activation rows per MMA (one TMEM lane each)
constexpr int kQBN = 256;                 // weight rows per tile
constexpr int kQBK = 64;                  // K per ring stage (128 bytes of 16-bit values)
constexpr int kQStages = 3;
constexpr int kQSlots = 2;                // decoded weight tiles in flight
constexpr int kQABytes = kQBM * 128;      // one activation box
constexpr int kQCodeBytes = kQBN * 32;    // 256 rows x 64 codes
constexpr int kQScaleBytes = kQBN * 16;   // 256 rows x one 16-byte scale segment
constexpr int kQStageBytes = 2 * kQABytes + kQCodeBytes + kQScaleBytes;
constexpr int kQSlotBytes = kQBN * 128;   // decoded: 256 rows x 64 values x 2 bytes
constexpr int kQConvWarps = 8;
constexpr int kQThreads = (6 + kQConvWarps) * 32;
constexpr int kQMaxGroups = 1024 + 64;

struct QTile {
  int shared_idx;  // >= 0 for a shared expert
  int expert;      // logical routed expert (-1 for shared)
  int xrow0;       // first activation row of the group
  int n_cols;      // activation rows of the group
  int phys;
  int mp, n_idx;   // 256-row activation block, weight tile
};

// K values per scale block and bytes per scale, by format
template <int F>
struct Q4Fmt;
template <>
struct Q4Fmt<kMXFP4> {
  static constexpr int blk = 32, sbytes = 1;
  static constexpr bool bf16_ops = true;
};
template <>
struct Q4Fmt<kNVFP4> {
  static constexpr int blk = 16, sbytes = 1;
  static constexpr bool bf16_ops = false;
};
template <>
struct Q4Fmt<kINT4> {
  static constexpr int blk = 128, sbytes = 2;
  static constexpr bool bf16_ops = false;
};

// Instruction descriptor of kind::f16 with fp32 D; A and B both bf16 (1) or
// both fp16 (0) in bits 7-9 / 10-12, K-major; N >> 3 in bits 17-22, M >> 4 in
// bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Eight E2M1 codes (nibble i = K i of the word) -> four fp16 pairs in K order
// (2i, 2i+1) by table lookup on the integer pipe: a byte permute picks each
// magnitude's high byte from an 8-entry table (E2M1 magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6 are the fp16 values 0x0000 3800 3C00 3E00 4000 4200 4400
// 4600, whose low bytes are all zero), a second permute spreads them into
// the pairs, and the code's sign bit is moved to bit 15 / 31 of its pair.
__device__ __forceinline__ void e2m1x8_to_f16x8_lut(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t m = w & 0x77777777u;  // magnitude codes
  const uint32_t m2 = m >> 16;
  const uint32_t s8 = w & 0x88888888u;  // sign bits
  const uint32_t t = s8 << 4;           // sign of the even code of byte b in the msb of byte b
  const uint32_t hA = prmt(0x3E3C3800u, 0x46444240u, m), hB = prmt(0x3E3C3800u, 0x46444240u, m2);
  o[0] = prmt(hA, 0u, 0x1404u);
  o[1] = prmt(hA, 0u, 0x3424u);
  o[2] = prmt(hB, 0u, 0x1404u);
  o[3] = prmt(hB, 0u, 0x3424u);
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    // byte 1 <- byte b of t (even code's sign), byte 3 <- byte b of s8 (odd code's sign)
    const uint32_t sg = prmt(t, s8, (uint32_t)b * 0x11u | (uint32_t)(4 + b) * 0x1100u);
    o[b] |= sg & 0x80008000u;
  }
}

// fp16 pair -> bf16 pair after multiplying both by f (exact when the products
// have at most 8 significant bits and lie in bf16's range).
__device__ __forceinline__ uint32_t f16x2_scale_to_bf16x2(uint32_t h2, float f) {
  const __half2 h = *reinterpret_cast<const __half2*>(&h2);
  const float2 v = __half22float2(h);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.x * f, v.y * f);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Eight INT4 codes (nibble i = K i of the word) -> four fp16 pairs in K order
// (2i, 2i+1), each value q * s: the nibbles become the fp16 integers
// 1024 + (q + 8) (one byte permute and one XOR per pair), 1032 is subtracted
// (exact) and the pair multiplied by the fp16 group scale s2 (exact while
// q * s needs at most fp16's 11 significant bits within its range).
__device__ __forceinline__ void int4x8_to_f16x8_scaled(uint32_t w, uint32_t s2, uint32_t (&o)[4]) {
  const uint32_t ev = w & 0x0f0f0f0fu;          // nibbles 0, 2, 4, 6 (one per byte)
  const uint32_t od = (w >> 4) & 0x0f0f0f0fu;   // nibbles 1, 3, 5, 7
  const __half2 sub = __half2half2(__ushort_as_half((unsigned short)0x6408u));  // 1032
  const __half2 sc = *reinterpret_cast<const __half2*>(&s2);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // bytes (ev byte p, -, od byte p, -); the masked bytes become the 0x64 of 1024
    const uint32_t sel = (uint32_t)p * 0x11u | (uint32_t)(4 + p) * 0x1100u;
    uint32_t v = (__byte_perm(ev, od, sel) & 0x00ff00ffu) ^ 0x64086408u;
    __half2 h = *reinterpret_cast<__half2*>(&v);
    h = __hmul2(__hsub2(h, sub), sc);
    o[p] = *reinterpret_cast<uint32_t*>(&h);
  }
}

}  // namespace

template <bool kGateUp, int F>
__global__ void __launch_bounds__(kQThreads, 1) ffn_gemm_q4_kernel(const __grid_constant__ GemmQ4Args a) {
  using Fm = Q4Fmt<F>;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;                                  // kQStages x (A0 | A1 | codes | scales)
  uint8_t* slots = smem + kQStages * kQStageBytes;         // kQSlots x decoded weight tile
  uint64_t* full = reinterpret_cast<uint64_t*>(slots + kQSlots * kQSlotBytes);
  uint64_t* empty = full + kQStages;
  uint64_t* dfull = empty + kQStages;
  uint64_t* dempty = dfull + kQSlots;
  uint64_t* acc_full = dempty + kQSlots;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_ngroups = reinterpret_cast<int*>(s_tmem + 2);
  int* s_gtile = s_ngroups + 2;                   // [kQMaxGroups + 1] first m-pair of each group (prefix)
  int* s_gexpert = s_gtile + kQMaxGroups + 1;     // [kQMaxGroups] routed expert, or -1 - shared index

  const int n_tiles_n = kGateUp ? a.N / 128 : a.N / kQBN;
  const int ksteps = a.K / kQBK;
  const int E = a.E;

  if (tid == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1 + kQConvWarps);  // the MMAs' commit + every converter warp
    }
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&dfull[i], kQConvWarps);
      mbar_init(&dempty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  pdl_wait_and_trigger();
  // Group table: shared experts first, then routed experts with rows, each
  // with its number of 256-row activation blocks (non-resident experts none).
  if (warp == 0) {
    int ng = 0, tiles = 0;
    for (int s = 0; s < a.n_shared; ++s) {
      if (lane == 0) {
        s_gtile[ng] = tiles;
        s_gexpert[ng] = -1 - s;
      }
      ++ng;
      tiles += ceil_div(a.T, 2 * kQBM);
    }
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int mt = 0;
      if (e < E) {
        const int cnt = __ldg(a.offsets + e + 1) - __ldg(a.offsets + e);
        const int p = a.slot_map ? __ldg(a.slot_map + e) : e;
        bool ok = cnt > 0;
        if (ok && (p < 0 || p >= a.n_phys)) {
          if (!(p == -1 && a.slot_map)) set_status(MOE_ERR_DEVICE_INDEX);
          ok = false;
        }
        mt = ok ? ceil_div(cnt, 2 * kQBM) : 0;
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
    tc::tmem_alloc(s_tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const int ngroups = *s_ngroups;
  const int total_tiles = s_gtile[ngroups] * n_tiles_n;

  auto decode = [&](int t) {
    QTile ti;
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_gtile[mid] * n_tiles_n <= t) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int mpg = s_gtile[g + 1] - s_gtile[g];
    const int local = t - s_gtile[g] * n_tiles_n;
    ti.n_idx = local / mpg;
    ti.mp = local - ti.n_idx * mpg;
    const int ex = s_gexpert[g];
    if (ex < 0) {
      ti.shared_idx = -1 - ex;
      ti.expert = -1;
      ti.xrow0 = a.T * a.k + ti.shared_idx * a.T;
      ti.n_cols = a.T;
      ti.phys = ti.shared_idx;
    } else {
      ti.shared_idx = -1;
      ti.expert = ex;
      ti.xrow0 = __ldg(a.offsets + ex);
      ti.n_cols = __ldg(a.offsets + ex + 1) - ti.xrow0;
      ti.phys = a.slot_map ? __ldg(a.slot_map + ex) : ex;
    }
    return ti;
  };

  if (warp == 0) {
    // ============================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(&a.tm_a);
      prefetch_tmap(&a.tm_w);
      prefetch_tmap(&a.tm_s);
      if (a.n_shared) {
        prefetch_tmap(&a.tm_wsh);
        prefetch_tmap(&a.tm_ssh);
      }
      const uint64_t pol = l2_evict_last_policy();  // both operands are re-read by other tiles
      uint32_t cnt = 0;
      for (int t = blockIdx.x; t < total_tiles && !*s_abort; t += gridDim.x) {
        const QTile ti = decode(t);
        const CUtensorMap* tw = ti.shared_idx >= 0 ? &a.tm_wsh : &a.tm_w;
        const CUtensorMap* ts = ti.shared_idx >= 0 ? &a.tm_ssh : &a.tm_s;
        const int arow = ti.xrow0 + ti.mp * 2 * kQBM;
        const int n0 = ti.n_idx * (kGateUp ? 128 : kQBN);
        const int r1 = kGateUp ? a.N + n0 : n0 + 128;  // weight rows of the second box
        for (int ks = 0; ks < ksteps; ++ks) {
          const int s = cnt % kQStages;
          if (!mbar_wait(&empty[s], ((cnt / kQStages) & 1u) ^ 1u)) {
            *s_abort = 1;
            break;
          }
          uint8_t* st = stages + s * kQStageBytes;
          mbar_arrive_expect_tx(&full[s], kQStageBytes);
          tma_load_2d(st, &a.tm_a, ks * 128, arow, &full[s], pol);
          tma_load_2d(st + kQABytes, &a.tm_a, ks * 128, arow + kQBM, &full[s], pol);
          uint8_t* sc = st + 2 * kQABytes;
          tma_load_3d(sc, tw, ks * 32, n0, ti.phys, &full[s], pol);
          tma_load_3d(sc + kQCodeBytes / 2, tw, ks * 32, r1, ti.phys, &full[s], pol);
          // the 16-byte scale segment holding this step's scales
          const int sx = ((ks * kQBK / Fm::blk) * Fm::sbytes) & ~15;
          uint8_t* ss = sc + kQCodeBytes;
          tma_load_3d(ss, ts, sx, n0, ti.phys, &full[s], pol);
          tma_load_3d(ss + kQScaleBytes / 2, ts, sx, r1, ti.phys, &full[s], pol);
          ++cnt;
        }
      }
      const uint32_t first = cnt > (uint32_t)kQStages ? cnt - kQStages : 0;
      for (uint32_t c = first; c < cnt; ++c) mbar_wait(&full[c % kQStages], (c / kQStages) & 1u);
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16kind(kQBM, kQBN, Fm::bf16_ops);
      uint32_t cnt = 0, dcnt = 0;
      int i = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < total_tiles && !*s_abort; t += gridDim.x, ++i) {
        const QTile ti = decode(t);
        const bool two = ti.n_cols - ti.mp * 2 * kQBM > kQBM;  // second activation half has rows
        if (!mbar_wait(acc_empty, ((uint32_t)i & 1u) ^ 1u)) {
          *s_abort = 1;
          break;
        }
        tc::fence_after_sync();
        for (int ks = 0; ks < ksteps; ++ks) {
          const int s = cnt % kQStages;
          const int j = dcnt % kQSlots;
          if (!mbar_wait(&full[s], (cnt / kQStages) & 1u) || !mbar_wait(&dfull[j], (dcnt / kQSlots) & 1u)) {
            *s_abort = 1;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa = smem_u32(stages + s * kQStageBytes);
          const uint32_t sb = smem_u32(slots + j * kQSlotBytes);
#pragma unroll
          for (int kk = 0; kk < kQBK / 16; ++kk) {
            const uint64_t bdesc = tc::kmajor_sw128_desc(sb + kk * 32);
            const uint32_t acc = (ks | kk) != 0 ? 1u : 0u;
            tc::mma_bf16(tmem_base, tc::kmajor_sw128_desc(sa + kk * 32), bdesc, idesc, acc);
            if (two) tc::mma_bf16(tmem_base + kQBN, tc::kmajor_sw128_desc(sa + kQABytes + kk * 32), bdesc, idesc, acc);
          }
          tc::commit(&empty[s]);   // the activation boxes are free once these MMAs have read them
          tc::commit(&dempty[j]);  // and so is the decoded weight tile
          issued = true;
          ++cnt;
          ++dcnt;
        }
        if (*s_abort) break;
        tc::commit(acc_full);
      }
      if (issued) {
        tc::commit(drain);
        mbar_wait(drain, 0);
      }
    }
  } else if (warp < 6) {
    // ============================================================== epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int i = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++i) {
      if (*s_abort || !mbar_wait(acc_full, (uint32_t)i & 1u)) {
        *s_abort = 1;
        break;
      }
      tc::fence_after_sync();
      const QTile ti = decode(t);
      float gsc = 1.f;
      if constexpr (F == kNVFP4) gsc = ti.shared_idx >= 0 ? __ldg(a.gsc_sh + ti.shared_idx) : __ldg(a.gsc + ti.expert);
      for (int h2 = 0; h2 < 2; ++h2) {
        const int m = ti.mp * 2 * kQBM + h2 * kQBM + r;  // row inside the group
        if (h2 == 1 && ti.n_cols - ti.mp * 2 * kQBM <= kQBM) break;  // (warp-uniform)
        const bool valid = m < ti.n_cols;
        float f = gsc;
        if constexpr (!Fm::bf16_ops) {
          if (valid) f = ldexpf(f, __ldg(a.xexp + ti.xrow0 + m));
        }
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h2 * kQBN);
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
                const float g0 = __uint_as_float(gv[2 * j]) * f, g1 = __uint_as_float(gv[2 * j + 1]) * f;
                const float u0 = __uint_as_float(uv[2 * j]) * f, u1 = __uint_as_float(uv[2 * j + 1]) * f;
                const float hh0 = g0 / (1.f + __expf(-g0)) * u0;
                const float hh1 = g1 / (1.f + __expf(-g1)) * u1;
                __nv_bfloat162 hb = __floats2bfloat162_rn(hh0, hh1);
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
          o += ti.n_idx * kQBN;
#pragma unroll 1
          for (int j0 = 0; j0 < kQBN; j0 += 32) {
            uint32_t v[32];
            tc::ld_32x32b_x32(taddr + j0, v);
            tc::ld_wait();
            if (valid) {
              uint32_t packed[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                __nv_bfloat162 hb =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * f, __uint_as_float(v[2 * j + 1]) * f);
                packed[j] = *reinterpret_cast<uint32_t*>(&hb);
              }
              uint4* dst = reinterpret_cast<uint4*>(o + j0);
#pragma unroll
              for (int w = 0; w < 4; ++w)
                dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1], packed[4 * w + 2], packed[4 * w + 3]);
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  } else {
    // ============================================================== converters
    const int row = tid - 6 * 32;  // weight row of the tile (0..255)
    uint32_t cnt = 0, dcnt = 0;
    // 16-byte halves of the row's 32 code bytes, read in an order that keeps
    // the 8 rows of each quarter-warp on distinct banks
    const int hfirst = (row >> 2) & 1;
    const uint32_t sw = (uint32_t)(row & 7);
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      for (int ks = 0; ks < ksteps; ++ks) {
        const int s = cnt % kQStages;
        const int j = dcnt % kQSlots;
        if (*s_abort || !mbar_wait(&full[s], (cnt / kQStages) & 1u) ||
            !mbar_wait(&dempty[j], ((dcnt / kQSlots) & 1u) ^ 1u)) {
          *s_abort = 1;
          break;
        }
        const uint32_t st = smem_u32(stages + s * kQStageBytes);
        const uint32_t ca = st + 2 * kQABytes + row * 32;
        const uint4 c0 = lds128(ca + 16 * hfirst);
        const uint4 c1 = lds128(ca + 16 * (hfirst ^ 1));
        const uint32_t cw[8] = {hfirst ? c1.x : c0.x, hfirst ? c1.y : c0.y, hfirst ? c1.z : c0.z,
                                hfirst ? c1.w : c0.w, hfirst ? c0.x : c1.x, hfirst ? c0.y : c1.y,
                                hfirst ? c0.z : c1.z, hfirst ? c0.w : c1.w};
        // this step's scale bytes of the row: at byte (ks*64/blk*sbytes) mod 16 of its segment
        const int soff = ((ks * kQBK / Fm::blk) * Fm::sbytes) & 15;
        const uint32_t sword = lds32(st + 2 * kQABytes + kQCodeBytes + row * 16 + (soff & ~3));
        const uint32_t sbits = sword >> (8 * (soff & 3));
        const uint32_t dst = smem_u32(slots + j * kQSlotBytes) + row * 128;
#pragma unroll
        for (int g = 0; g < 8; ++g) {  // granule g: K = 8g .. 8g+7 of the step
          uint32_t o[4];
          if constexpr (F == kMXFP4) {
            // E8M0 scale of the 32-block holding this granule; E2M1 -> fp16 by
            // the hardware conversion, x 2^(e-127) in fp32, -> bf16 (exact:
            // 2 significant bits, bf16's exponent range)
            const float f = e8m0_to_f32((sbits >> (8 * (g >> 2))) & 0xffu);
            uint32_t h0, h1, h2, h3;
            e2m1x8_to_f16x8(cw[g], h0, h1, h2, h3);
            o[0] = f16x2_scale_to_bf16x2(h0, f);
            o[1] = f16x2_scale_to_bf16x2(h1, f);
            o[2] = f16x2_scale_to_bf16x2(h2, f);
            o[3] = f16x2_scale_to_bf16x2(h3, f);
          } else if constexpr (F == kNVFP4) {
            // E4M3 byte of the 16-block holding this granule, as an fp16 pair
            const uint32_t e = (sbits >> (8 * (g >> 1))) & 0xffu;
            const uint32_t s2 = e4m3x2_to_f16x2(e | (e << 8));
            e2m1x8_to_f16x8_lut(cw[g], o);
#pragma unroll
            for (int q = 0; q < 4; ++q) o[q] = hmul2_u32(o[q], s2);
          } else {
            // bf16 group scale (one per 128 K: the low 16 bits) as an fp16 pair
            const __half hs = __float2half_rn(bf16_bits_to_f32(sbits & 0xffffu));
            const __half2 hs2 = __half2half2(hs);
            int4x8_to_f16x8_scaled(cw[g], *reinterpret_cast<const uint32_t*>(&hs2), o);
          }
          // 128-byte swizzle: granule g of row r sits at granule g ^ (r & 7)
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst + (((uint32_t)g ^ sw) << 4)), "r"(o[0]),
                       "r"(o[1]), "r"(o[2]), "r"(o[3])
                       : "memory");
        }
        fence_proxy_async_smem();  // the MMA (async proxy) reads what these threads wrote
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&dfull[j]);
          mbar_arrive(&empty[s]);
        }
        ++cnt;
        ++dcnt;
      }
      if (*s_abort) break;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem_base, 512);
}

// ------------------------------------------------------------------ host side
bool gemm_q4_supported(int F, int N, int K, bool gate_up) {
  if (F != kMXFP4 && F != kNVFP4 && F != kINT4) return false;
  if (K % kQBK) return false;
  const int blk = F == kMXFP4 ? 32 : (F == kNVFP4 ? 16 : 128);
  const int sb = F == kINT4 ? 2 : 1;
  if (((K / blk) * sb) % 16) return false;  // TMA row pitch of the scale matrix
  return gate_up ? (N % 128 == 0) : (N % kQBN == 0);
}

bool gemm_q4_bf16_activations(int F) { return F == kMXFP4; }

template <bool GU, int F>
static cudaError_t launch_q4(const GemmQ4Args& a, int grid, size_t smem, cudaStream_t st) {
  auto kern = ffn_gemm_q4_kernel<GU, F>;
  {
    cudaError_t err = set_dyn_smem_once<ffn_gemm_q4_kernel<GU, F>>(smem);
    if (err != cudaSuccess) return err;
  }
  ProfScope prof(GU ? "ffn_gemm_q4_stage1_gate_up" : "ffn_gemm_q4_stage2_down", st);
  return launch_pdl(kern, dim3(grid), dim3(kQThreads), smem, st, a);
}

cudaError_t launch_ffn_gemm_q4(int F, bool gate_up, GemmQ4Args a, const GemmQ4Pointers& p, int n_sms,
                               int smem_max, cudaStream_t st, int* unsupported) {
  *unsupported = 0;
  const size_t smem = 1024 + (size_t)kQStages * kQStageBytes + (size_t)kQSlots * kQSlotBytes + 1024 +
                      (size_t)(2 * kQMaxGroups + 8) * 4;
  if ((int)smem > smem_max || !gemm_q4_supported(F, a.N, a.K, gate_up)) {
    *unsupported = 1;
    return cudaSuccess;
  }
  const int blk = F == kMXFP4 ? 32 : (F == kNVFP4 ? 16 : 128);
  const int sb = F == kINT4 ? 2 : 1;
  const uint64_t wrows = gate_up ? 2 * (uint64_t)a.N : (uint64_t)a.N;
  const uint64_t code_row = (uint64_t)a.K / 2, scale_row = (uint64_t)(a.K / blk) * sb;
  bool ok = true;
  {
    const uint64_t dims[2] = {(uint64_t)a.K * 2, (uint64_t)p.rows_total};
    const uint64_t strides[1] = {(uint64_t)a.K * 2};
    const uint32_t box[2] = {128, (uint32_t)kQBM};
    ok = ok && encode_tmap_u8(&a.tm_a, p.x, 2, dims, strides, box, true);
  }
  auto weights = [&](CUtensorMap* tw, CUtensorMap* ts, const void* w, int64_t sw, const void* s, int64_t ss,
                     uint64_t n) {
    const uint64_t wd[3] = {code_row, wrows, n};
    const uint64_t wst[2] = {code_row, (uint64_t)sw};
    const uint32_t wb[3] = {32, 128, 1};
    const uint64_t sd[3] = {scale_row, wrows, n};
    const uint64_t sst[2] = {scale_row, (uint64_t)ss};
    const uint32_t sbx[3] = {16, 128, 1};
    return encode_tmap_u8(tw, w, 3, wd, wst, wb, false) && encode_tmap_u8(ts, s, 3, sd, sst, sbx, false);
  };
  ok = ok && weights(&a.tm_w, &a.tm_s, p.w, p.stride_w, p.s, p.stride_s, (uint64_t)a.n_phys);
  if (a.n_shared > 0)
    ok = ok && weights(&a.tm_wsh, &a.tm_ssh, p.w_sh, p.stride_w_sh, p.s_sh, p.stride_s_sh, (uint64_t)a.n_shared);
  else {
    a.tm_wsh = a.tm_w;
    a.tm_ssh = a.tm_s;
  }
  if (!ok) {
    *unsupported = 1;
    return cudaSuccess;
  }
  const int n_tiles_n = gate_up ? a.N / 128 : a.N / kQBN;
  const long rows = (long)a.T * a.k;
  const long max_mp = (rows + 2 * kQBM - 1) / (2 * kQBM) + (a.E < rows ? a.E : rows) +
                      (long)a.n_shared * ((a.T + 2 * kQBM - 1) / (2 * kQBM));
  const long max_tiles = max_mp * n_tiles_n;
  const int grid = (int)(max_tiles < n_sms ? max_tiles : n_sms);
  if (grid < 1) return cudaSuccess;
  switch (F) {
    case kMXFP4: return gate_up ? launch_q4<true, kMXFP4>(a, grid, smem, st) : launch_q4<false, kMXFP4>(a, grid, smem, st);
    case kNVFP4: return gate_up ? launch_q4<true, kNVFP4>(a, grid, smem, st) : launch_q4<false, kNVFP4>(a, grid, smem, st);
    default: return gate_up ? launch_q4<true, kINT4>(a, grid, smem, st) : launch_q4<false, kINT4>(a, grid, smem, st);
  }
}

}  // namespace moe
