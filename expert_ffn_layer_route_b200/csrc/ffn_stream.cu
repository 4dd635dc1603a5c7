// Grouped SwiGLU expert FFN, weight-streaming form (decode and small groups).
//
// During decode each new token reads the weights of its active experts
// ("Mixture of experts VRAM: total vs active parameters", section "What
// active parameters change"), and with a batch the tokens of one step go to
// different experts, so a step touches many experts; grouping the tokens
// that chose the same expert lets one weight read serve all of them
// ("Understanding MoE Inference Costs on Galactus", section "Prompt
// processing is a different phase").  This kernel therefore walks work items
// (expert, row tile) and streams each tile's weight rows from HBM exactly once
// per pass of up to 32 of the expert's rows, applying them to all of those
// rows at once.  The expert's gate / up / down projections (FloE verdict
// page, JSON field referee_report.summary) are applied as SwiGLU:
//   stage 1: h = silu(x W_gate^T) * (x W_up^T)   (gate and up tiles paired)
//   stage 2: y = h W_down^T
//
// Block = 8 consumer warps + 1 producer warp, three blocks per SM when a pass
// takes one group of 8 activation rows (else two), persistent over the work
// items (dynamically claimed when there are more than three per block).  The
// producer's elected lane issues TMA tiled loads
// (128-row x 128-byte boxes, 128-byte swizzle) of the weights and of the
// expert's activation rows into a ring of shared-memory stages, completing on
// mbarriers.  Consumers decode the 4-bit codes to fp16 (E2M1 with the
// hardware cvt; INT4 as offset integers 1024 + 16^j (q + 8), one AND-XOR per
// pair, whose constant part is removed per scale group) and run m16n8k16 MMAs
// with fp32 accumulation.  Block scales: MXFP4 (E8M0 per 32) and INT4 (bf16
// per 128) multiply the fp32 partial sums of their block; NVFP4 (E4M3 per 16)
// multiplies the fp16 weights (exact in fp16) and its fp32 global scale is
// applied in the epilogue.  An item's block scales cross the stage ring once
// and stay in tensor memory (TMEM) while the item runs, each consumer lane
// holding one weight row's.  Within each 32-wide K block lane c of a quad
// holds K = 8c..8c+7, i.e. the MMA's K order is a fixed permutation of the
// block, applied identically to both operands.  Activation rows (and bf16
// weight rows) are read through the row order sigma(g) = (g>>1) | (g&1)<<2
// inside each group of 8 so that the swizzled 16-byte reads are free of bank
// conflicts; the epilogue maps columns (rows) back through the same sigma.
// A full K chunk runs as straight-line code (every block and column group
// known at compile time); only a ragged last chunk takes the guarded path.
#include <cstdlib>
#include <type_traits>

#include "ffn_stream.cuh"
#include "tc_ptx.cuh"
#include "launch.cuh"
#include "profile.cuh"

namespace moe {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kRowsPerStage = 256;  // smem weight rows per stage (2 boxes of 128)
constexpr int kBoxRows = 128;
constexpr int kLine = 128;          // bytes per smem row (one swizzle line)
constexpr int kMaxStages = 8;

template <int F>
struct FmtTraits;
template <>
struct FmtTraits<kBF16> {
  static constexpr int kc = 64;     // K values per stage (128 bytes of a weight row)
  static constexpr int blk = 0;     // scale block (0: none)
  static constexpr int sbytes = 0;  // bytes per scale
  static constexpr int kcpc = 1;    // 32-bit TMEM columns of scales per stage (unused without scales)
};
template <>
struct FmtTraits<kMXFP4> {
  static constexpr int kc = 256, blk = 32, sbytes = 1, kcpc = 2;
};
template <>
struct FmtTraits<kNVFP4> {
  static constexpr int kc = 256, blk = 16, sbytes = 1, kcpc = 4;
};
template <>
struct FmtTraits<kINT4> {
  static constexpr int kc = 256, blk = 128, sbytes = 2, kcpc = 1;
};

__device__ __forceinline__ int sigma8(int g) { return (g >> 1) | ((g & 1) << 2); }

// Position in the ring of shared-memory stages: the stage index and the
// parity of its current fill, advanced without dividing by the run-time ring
// depth (a division per K chunk costs the consumers' integer pipe ~20
// instructions twice over).
struct RingPos {
  int s;
  uint32_t ph;
  int n;
  __device__ __forceinline__ void next() {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// Shared-memory header: barriers, flags, offsets [E+1], group table.
__host__ __device__ constexpr int stream_hdr_bytes(int E, int n_shared) {
  return ((16 * kMaxStages + 64 + 4 * ((E + 4) + 2 * (E + n_shared + 4))) + 1023) & ~1023;
}

// Everything a block needs to know about one work item.
struct Item {
  int valid;
  int shared_idx;  // >= 0 for a shared expert
  int tile;
  int xrow0;       // first activation / output row of this expert
  int n_cols;      // activation rows of this expert
  int phys;        // physical expert index (TMA coordinate)
  int pass;        // which XCOLS-wide slice of the expert's rows
  const uint8_t* sbase;
  float gscale;
};

// Work items are (group, tile, pass): groups are the shared experts then the
// routed experts with rows (gitem holds each group's first item), and every
// pass of XCOLS activation rows is its own item, passes fastest, so that the
// CTAs streaming one weight tile for different passes run side by side and
// share it through L2.
template <int F>
__device__ __forceinline__ Item decode_item(const FfnArgs& a, int item, int ntile, const int* gitem,
                                            const int* gexp, int ngroups, const int* offs) {
  Item it{};
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (gitem[mid] <= item) lo = mid; else hi = mid - 1;
  }
  const int passes = (gitem[lo + 1] - gitem[lo]) / ntile;
  const int local = item - gitem[lo];
  it.tile = local / passes;
  it.pass = local - it.tile * passes;
  it.valid = 1;
  const int ex = gexp[lo];
  const int grp = ex < 0 ? -1 - ex : a.n_shared + ex;
  if (ex < 0) {
    it.shared_idx = grp;
    it.xrow0 = a.T * a.k + grp * a.T;
    it.n_cols = a.T;
    it.phys = grp;
    it.sbase = a.s_sh ? a.s_sh + (int64_t)grp * a.stride_s_sh : nullptr;
    it.gscale = (F == kNVFP4 && a.gsc_sh) ? __ldg(a.gsc_sh + grp) : 1.f;
  } else {
    const int e = ex;
    it.shared_idx = -1;
    it.xrow0 = offs[e];
    it.n_cols = offs[e + 1] - offs[e];
    int p = a.slot_map ? __ldg(a.slot_map + e) : e;
    if (p == -1 && a.slot_map) {
      it.valid = 0;  // not resident in this call: skipped
      p = 0;
    } else if (p < 0 || p >= a.n_phys || it.xrow0 < 0 || it.n_cols < 0 || it.xrow0 + it.n_cols > a.T * a.k) {
      set_status(MOE_ERR_DEVICE_INDEX);
      it.valid = 0;
      p = 0;
    }
    it.phys = p;
    it.sbase = a.s ? a.s + (int64_t)p * a.stride_s : nullptr;
    it.gscale = (F == kNVFP4 && a.gsc) ? __ldg(a.gsc + e) : 1.f;
  }
  return it;
}

template <int F, int NG, bool kGateUp, int MINB, bool kHalf, bool kSplit>
__global__ void __launch_bounds__(kThreads, MINB) ffn_stream_kernel(const __grid_constant__ FfnArgs a) {
  using Tr = FmtTraits<F>;
  constexpr int KC = Tr::kc;
  constexpr int XCOLS = NG * 8;                 // activation rows per pass
  constexpr int NXBOX = (KC * 2) / kLine;       // 128-byte activation boxes per stage
  // Item geometry.  Full items: 128 gate + 128 up rows (stage 1) or 256 rows
  // (stage 2), two m16 tiles per consumer warp.  Half items (kHalf, for
  // batches whose items would not fill the grid): 64 + 64 or 128 rows, one
  // m16 tile per warp -- in stage 1 its rows g are gate rows and its rows g+8
  // the up rows of the same outputs.
  constexpr int kMT = kHalf ? 1 : 2;                                             // m16 tiles per warp
  constexpr int kItemRows = kGateUp ? (kHalf ? 64 : 128) : (kHalf ? 128 : 256);  // output rows per item
  constexpr int kWarpRows = kItemRows / kConsumerWarps;                          // output rows per warp
  constexpr int W_BYTES = (kGateUp ? 2 * kItemRows : kItemRows) * kLine;
  constexpr int X_BYTES = NXBOX * XCOLS * kLine;
  constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  constexpr int kCpc = Tr::kcpc;                // TMEM scale columns per K chunk
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA destinations
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);
  int* s_ngroups = reinterpret_cast<int*>(empty + kMaxStages) + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(empty + kMaxStages) + 2;
  volatile int* s_hdr = reinterpret_cast<volatile int*>(empty + kMaxStages) + 4;  // [kMaxStages] item of a stage
  int* s_offs = reinterpret_cast<int*>(empty + kMaxStages) + 16;                  // [E+1]
  int* s_gitem = s_offs + (a.E + 4);                             // [groups+1]
  int* s_gexp = s_gitem + (a.E + a.n_shared + 4);                // [groups]
  uint8_t* s_stage = smem + stream_hdr_bytes(a.E, a.n_shared);

  const int E = a.E;
  if (tid == 0) {
    for (int i = 0; i < a.n_stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  pdl_wait_and_trigger();
  for (int i = tid; i <= E; i += kThreads) s_offs[i] = __ldg(a.offsets + i);
  __syncthreads();
  const int rows_per_item = kItemRows;
  const int ntile = ceil_div(a.N, rows_per_item);
  if (warp == 0) {
    // Block scales live in tensor memory while an item runs: lane i of warp w
    // keeps the scales of one weight row in TMEM lane 32 (w % 4) + i, columns
    // [(w / 4) C, (w / 4 + 1) C); an SM's blocks together take <= 512 columns.
    if (Tr::blk) {
      tc::tmem_alloc(s_tmem, (uint32_t)a.tmem_alloc);
      tc::tmem_relinquish();
    }
    int ng = 0, items = 0;
    for (int sh = 0; sh < a.n_shared; ++sh) {
      if (lane == 0) {
        s_gitem[ng] = items;
        s_gexp[ng] = -1 - sh;
      }
      ++ng;
      items += ntile * ceil_div(a.T, XCOLS);
    }
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int cnt_items = 0;
      if (e < E) {
        const int r0e = s_offs[e], cnt = s_offs[e + 1] - r0e;
        const int p = a.slot_map ? __ldg(a.slot_map + e) : e;
        bool ok = cnt > 0;
        if (ok && (p < 0 || p >= a.n_phys || r0e < 0 || r0e + cnt > a.T * a.k)) {
          if (!(p == -1 && a.slot_map)) set_status(MOE_ERR_DEVICE_INDEX);  // -1: not resident, skipped
          ok = false;
        }
        cnt_items = ok ? ntile * ceil_div(cnt, XCOLS) : 0;
      }
      const uint32_t on = __ballot_sync(0xffffffffu, cnt_items > 0);
      int incl = cnt_items;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (cnt_items > 0) {
        const int slot = ng + __popc(on & ((1u << lane) - 1u));
        s_gitem[slot] = items + incl - cnt_items;
        s_gexp[slot] = e;
      }
      ng += __popc(on);
      items += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_gitem[ng] = items;
      *s_ngroups = ng;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int ngroups = *s_ngroups;
  const int n_items = s_gitem[ngroups];
  // split K (one column group only): item i of the launch is slice i % S of
  // item i / S; every block sees the same n_items, so a launch whose items
  // would overflow the partial buffers runs unsplit everywhere
  int S = (kSplit && NG == 1) ? a.split : 1;
  if (S > 1 && (int64_t)n_items * S > a.split_cap) S = 1;
  const int n_work = n_items * S;
  const int K = a.K;
  const int srow = Tr::blk ? (K / Tr::blk) * Tr::sbytes : 0;
  const int nchunks = ceil_div(K, KC);
  const int nstage = a.n_stages;
  const int n_sslots = Tr::blk ? a.n_sslots : 0;  // ring stages carrying an item's block scales
  const int slot_warps = kConsumerWarps / (n_sslots ? n_sslots : 1);
  const int x_row_bytes = K * 2;
  // Block b starts with item b.  With more than three items per block the
  // items after the first gridDim.x are claimed one at a time from a
  // launch-wide counter (zeroed before the launch), so that blocks that run
  // faster take more of them (Kimi T=128: 1.35 vs 1.41 ms per layer); the
  // first ring stage of every item then carries its index in s_hdr for the
  // consumers, and a last stage with index -1 ends the work.  With fewer,
  // block b takes items b, b + gridDim.x, ... and consumers follow the same
  // sequence on their own (the claims cost more than the balance gained:
  // gpt-oss stage 2 at T=64, 2.97 items per block, 114 vs 108 us).
  const bool dynamic = n_work > 3 * (int)gridDim.x;

  if (warp == kConsumerWarps) {
    // ===================================================== producer warp
    if (lane == 0) {
      prefetch_tmap(&a.tm_w);
      prefetch_tmap(&a.tm_x);
      if (a.n_shared) prefetch_tmap(&a.tm_wsh);
      const uint64_t pol_w = a.w_l2_first ? l2_evict_first_policy() : l2_evict_normal_policy();
      const uint64_t pol_x = l2_evict_last_policy();
      uint32_t cnt = 0;
      RingPos rp{0, 0u, nstage};
      int item = blockIdx.x;
      while (item < n_work && !*s_abort) {
        int next_item = n_work;
        const int base = item / S, slice = item - base * S;
        const int ch_lo = slice * nchunks / S, ch_hi = (slice + 1) * nchunks / S;
        // claim a ring's depth (+1) ahead of the item's end: the answer is back
        // before the producer needs it, and the claimed item waits only that long
        const int claim_at = max(ch_lo, ch_hi - 1 - nstage);
        const Item it = decode_item<F>(a, base, ntile, s_gitem, s_gexp, ngroups, s_offs);
        const int r0 = it.tile * rows_per_item;
        const int nrows = min(rows_per_item, a.N - r0);
        const CUtensorMap* tw = it.shared_idx >= 0 ? &a.tm_wsh : &a.tm_w;
        // The item's block scales first, in n_sslots ring stages: stage j holds
        // the rows of consumer warps [j * slot_warps, (j + 1) * slot_warps) --
        // gate rows then up rows (stage 1), or kWarpRows rows per warp (stage 2)
        // -- each a contiguous range of the row-major scale matrix.
        for (int j = 0; j < n_sslots && !*s_abort; ++j) {
          const int s = rp.s;
          if (!mbar_wait(&empty[s], rp.ph ^ 1u)) {
            *s_abort = 1;
            break;
          }
          s_hdr[s] = item;
          uint8_t* dst = s_stage + s * STAGE_BYTES;
          const int wrows = kWarpRows;  // scale rows per warp and matrix half
          const int first = j * slot_warps * wrows;
          const int cnt_rows = max(0, min(nrows - first, slot_warps * wrows));
          const uint32_t bytes = (uint32_t)(cnt_rows * srow);
          mbar_arrive_expect_tx(&full[s], it.valid ? bytes * (kGateUp ? 2u : 1u) : 0u);
          if (it.valid && cnt_rows > 0) {
            bulk_g2s(dst, it.sbase + (int64_t)(r0 + first) * srow, bytes, &full[s]);
            if (kGateUp)
              bulk_g2s(dst + slot_warps * wrows * srow, it.sbase + (int64_t)(a.N + r0 + first) * srow, bytes,
                       &full[s]);
          }
          ++cnt;
          rp.next();
        }
        // boxes of weight rows: stage 1 gate rows r0.. and up rows N+r0..; stage 2 rows r0.., r0+128..
        const int nbox_w = kGateUp ? 2 : (!kHalf && nrows > kBoxRows ? 2 : 1);
        constexpr int kBoxH = kGateUp ? kItemRows : kBoxRows;  // rows per weight box
        const int c0 = it.pass * XCOLS;
        for (int ch = ch_lo; ch < ch_hi && !*s_abort; ++ch) {
          if (ch == claim_at) next_item = dynamic ? (int)gridDim.x + atomicAdd(a.work_ctr, 1) : item + (int)gridDim.x;
          const int s = rp.s;
          if (!mbar_wait(&empty[s], rp.ph ^ 1u)) {
            *s_abort = 1;
            break;
          }
          s_hdr[s] = item;
          uint8_t* st_w = s_stage + s * STAGE_BYTES;
          uint8_t* st_x = st_w + W_BYTES;
          const int kb = ch * kLine;                 // byte offset inside a weight row
          const int xb0 = ch * KC * 2;               // byte offset inside an activation row
          int nxb = 0;
          for (int q = 0; q < NXBOX; ++q) nxb += (xb0 + q * kLine < x_row_bytes) ? 1 : 0;
          const uint32_t bytes = it.valid ? (uint32_t)(nbox_w * kBoxH * kLine + nxb * XCOLS * kLine) : 0u;
          mbar_arrive_expect_tx(&full[s], bytes);
          if (it.valid) {
            if (kGateUp) {
              tma_load_3d(st_w, tw, kb, r0, it.phys, &full[s], pol_w);
              tma_load_3d(st_w + kItemRows * kLine, tw, kb, a.N + r0, it.phys, &full[s], pol_w);
            } else {
              tma_load_3d(st_w, tw, kb, r0, it.phys, &full[s], pol_w);
              if (nbox_w == 2) tma_load_3d(st_w + kBoxRows * kLine, tw, kb, r0 + kBoxRows, it.phys, &full[s], pol_w);
            }
            for (int q = 0; q < nxb; ++q)
              tma_load_2d(st_x + q * XCOLS * kLine, &a.tm_x, xb0 + q * kLine, it.xrow0 + c0, &full[s], pol_x);
          }
          ++cnt;
          rp.next();
        }
        item = next_item;
      }
      // end of work: one more stage whose header says so
      if (dynamic && !*s_abort) {
        const int s = rp.s;
        if (mbar_wait(&empty[s], rp.ph ^ 1u)) {
          s_hdr[s] = -1;
          mbar_arrive(&full[s]);
          ++cnt;
        } else {
          *s_abort = 1;
        }
      }
      // Let every load this lane issued land before the block can exit.
      const uint32_t first = cnt > (uint32_t)nstage ? cnt - nstage : 0;
      for (uint32_t c = first; c < cnt; ++c) mbar_wait(&full[c % nstage], (c / nstage) & 1u);
    }
    return;
  }

  // ======================================================= consumer warps
  const int g = lane >> 2, c = lane & 3;
  const int sg = sigma8(g);
  // Rows of this warp's m16 tile(s) inside a stage (multiples of 8).
  const int m0 = warp * kWarpRows;  // stage 1: this warp's gate rows; stage 2: its first row
  constexpr int kDm = kGateUp ? kItemRows : 16;  // full items: second m-tile, rows below the first
  // Stage-relative byte offsets of this lane's operands.  A 128-byte row r
  // keeps its 16-byte granule j at ((j ^ (r & 7)) << 4) (TMA 128-byte
  // swizzle).  For every row this lane reads, r & 7 is g (4-bit codes) or
  // sigma(g) (bf16 weights, activations), so the granule of block b is one XOR
  // away from the lane's block-0 address, and rows g + 8 and the second
  // m-tile sit at fixed distances from it.
  const uint32_t w_lane = (F == kBF16) ? (uint32_t)(m0 + sg) * kLine + ((uint32_t)(c ^ sg) << 4)
                                       : (uint32_t)(m0 + g) * kLine + ((uint32_t)g << 4) + 4u * c;
  // A-fragment rows g -> g + 8: the next 8 rows, or (half stage 1) the up rows
  constexpr uint32_t kRow8 = (kGateUp && kHalf) ? kItemRows * kLine : 8 * kLine;
  constexpr uint32_t kDmBytes = kDm * kLine;
  const uint32_t x_lane = W_BYTES + (uint32_t)sg * kLine + ((uint32_t)(c ^ sg) << 4);
  // Block scales: lane c of a quad owns the scale row of m-tile c>>1, row
  // g + 8(c&1) (each lane of the warp a different row), keeps it in TMEM, and
  // hands the quad's other lanes what they need through shuffles.
  const uint32_t t_row = Tr::blk ? *s_tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((warp >> 2) * a.tmem_cols)
                                 : 0u;
  // the owned row inside its scale stage (gate rows of the stage's warps, then up rows)
  const int s_wl = warp % slot_warps;
  const int s_slot = warp / slot_warps;  // the scale stage that carries this warp's rows
  // (half items own two rows per quad: lanes c and c+2 hold the same one)
  const int s_row = kHalf ? (kGateUp ? ((c & 1) ? kWarpRows * slot_warps : 0) + kWarpRows * s_wl + g
                                     : kWarpRows * s_wl + g + 8 * (c & 1))
                          : (kGateUp ? ((c >> 1) ? kWarpRows * slot_warps : 0) + kWarpRows * s_wl + g + 8 * (c & 1)
                                     : kWarpRows * s_wl + 16 * (c >> 1) + g + 8 * (c & 1));
  RingPos rc{0, 0u, nstage};
  const uint32_t stage0 = smem_u32(s_stage);
  for (int item = blockIdx.x;; item += gridDim.x) {
    if (dynamic) {
      // the item's first stage names it (or the end of work); the loops
      // below wait on it again: that phase is complete and cannot move on
      // before this warp releases the stage
      const int s = rc.s;
      if (*s_abort || !mbar_wait(&full[s], rc.ph)) {
        *s_abort = 1;
        break;
      }
      item = s_hdr[s];
      if (item < 0) break;
    } else if (item >= n_work) {
      break;
    }
    const int base = item / S, slice = item - base * S;
    const int ch_lo = slice * nchunks / S, ch_hi = (slice + 1) * nchunks / S;
    const Item it = decode_item<F>(a, base, ntile, s_gitem, s_gexp, ngroups, s_offs);
    const int r0 = it.tile * rows_per_item;
    const int nrows = min(rows_per_item, a.N - r0);
    const bool active = it.valid && m0 < nrows;
    const int c0 = it.pass * XCOLS;
    const int ncols = min(XCOLS, it.n_cols - c0);
    const int ng_act = ceil_div(ncols, 8);
    // --------------------------------------------- block scales -> TMEM
    for (int j = 0; j < n_sslots; ++j) {
      const int s = rc.s;
      if (*s_abort || !mbar_wait(&full[s], rc.ph)) {
        *s_abort = 1;
        break;
      }
      if (active && ncols > 0 && s_slot == j) {
        const uint32_t ra = stage0 + s * STAGE_BYTES + s_row * srow;
        for (int cb = 0; cb < a.tmem_cols; cb += 4) {
          uint32_t v[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int b0 = 4 * (cb + t);
            if (b0 + 4 <= srow) {
              if ((srow & 3) == 0) v[t] = lds32(ra + b0);
              else if ((srow & 1) == 0) v[t] = lds16(ra + b0) | (lds16(ra + b0 + 2) << 16);
              else v[t] = lds8(ra + b0) | (lds8(ra + b0 + 1) << 8) | (lds8(ra + b0 + 2) << 16) | (lds8(ra + b0 + 3) << 24);
            } else {
              v[t] = 0;
              for (int u = 0; u < 4 && b0 + u < srow; ++u) v[t] |= lds8(ra + b0 + u) << (8 * u);
            }
          }
          tc::tmem_st_32x32b_x4(t_row + cb, v);
        }
        tc::tmem_st_wait();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      rc.next();
    }
    if (*s_abort) break;
    float acc[NG][kMT][4];
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[q][mt][r] = 0.f;
    float tmp[NG][kMT][4];  // INT4 group partials
    float gbias[NG][2];   // INT4 constant part of the group's partials, per column
    const int n_grp = K / 128;
    // INT4: where this lane's columns' constant parts start (row * n_grp), once per item
    [[maybe_unused]] int gb_off[NG][2];
    if constexpr (F == kINT4) {
#pragma unroll
      for (int q = 0; q < NG; ++q)
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int col = c0 + q * 8 + sigma8(2 * c + hc);
          gb_off[q][hc] = (it.xrow0 + (col < it.n_cols ? col : 0)) * n_grp;
        }
    }
    for (int ch = ch_lo; ch < ch_hi; ++ch) {
      const int s = rc.s;
      const bool work = active && ncols > 0;
      // this chunk's scales of the owned row (issued before the wait for the stage)
      uint32_t sv[4] = {0u, 0u, 0u, 0u};
      if constexpr (Tr::blk != 0) {
        if (work) tc::tmem_ld_cols<kCpc>(t_row + ch * kCpc, sv);
      }
      if (*s_abort || !mbar_wait(&full[s], rc.ph)) {
        if constexpr (Tr::blk != 0) {
          if (work) tc::tmem_ld_wait<kCpc>(sv);
        }
        *s_abort = 1;
        break;
      }
      if (work) {
        if constexpr (Tr::blk != 0) tc::tmem_ld_wait<kCpc>(sv);
        const uint32_t wst = stage0 + s * STAGE_BYTES;
        const uint32_t wa0 = wst + w_lane;
        const uint32_t xa0 = wst + x_lane;  // activation granule of even blocks
        const uint32_t xa1 = xa0 ^ 64u;     // odd blocks: granule 4 + c
        const int nblk = min(KC, K - ch * KC) / 32;
        // MXFP4: the owned row's eight scales of this chunk, as fp32
        float sc8[KC / 32];
        if constexpr (F == kMXFP4) {
#pragma unroll
          for (int p = 0; p < KC / 64; ++p) e8m0x2_to_f32x2((sv[p >> 1] >> (16 * (p & 1))) & 0xffffu, sc8[2 * p], sc8[2 * p + 1]);
        }
        // One 32-wide K block b for NQ column groups; with kGuard the groups
        // at or beyond ng_act are skipped at run time.
        auto block = [&](const int b, auto nq_tag, auto guard_tag) {
          constexpr int NQ = decltype(nq_tag)::value;
          constexpr bool kGuard = decltype(guard_tag)::value;
          [[maybe_unused]] float scb[kMT][2];  // MXFP4 scale of block b for [m-tile][row g / g+8]
          if constexpr (F == kMXFP4) {
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
              for (int hr = 0; hr < 2; ++hr)
                scb[mt][hr] = __shfl_sync(0xffffffffu, sc8[b], (lane & ~3) | (2 * mt + hr));
          }
          uint32_t A[kMT][2][4];  // [m-tile][k16 tile][reg]
          if constexpr (F == kBF16) {
            const uint32_t wa = wa0 ^ ((uint32_t)b << 6);
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
              const uint4 lo = lds128(wa + mt * kDmBytes);
              const uint4 hi = lds128(wa + mt * kDmBytes + kRow8);
              A[mt][0][0] = lo.x; A[mt][0][1] = hi.x; A[mt][0][2] = lo.y; A[mt][0][3] = hi.y;
              A[mt][1][0] = lo.z; A[mt][1][1] = hi.z; A[mt][1][2] = lo.w; A[mt][1][3] = hi.w;
            }
          } else {
            const uint32_t wa = wa0 ^ ((uint32_t)b << 4);
            // NVFP4: the two 16-block scales of block b of each owned row sit in
            // one 16-bit half of the row's chunk word b>>1; this lane's 8 values
            // lie in 16-block 2b + (c>>1)
            [[maybe_unused]] uint32_t nv[kMT][2];
            if constexpr (F == kNVFP4) {
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr)
                  nv[mt][hr] = __shfl_sync(0xffffffffu, sv[b >> 1], (lane & ~3) | (2 * mt + hr)) >>
                               (16 * (b & 1) + 8 * (c >> 1));
            }
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
              const uint32_t wlo = lds32(wa + mt * kDmBytes);
              const uint32_t whi = lds32(wa + mt * kDmBytes + kRow8);
              uint32_t l0, l1, l2, l3, h0, h1, h2, h3;
              if constexpr (F == kINT4) {
                int4x8_to_f16x8_offset(wlo, l0, l1, l2, l3);
                int4x8_to_f16x8_offset(whi, h0, h1, h2, h3);
              } else {
                e2m1x8_to_f16x8(wlo, l0, l1, l2, l3);
                e2m1x8_to_f16x8(whi, h0, h1, h2, h3);
              }
              if constexpr (F == kNVFP4) {
                const uint32_t pair = (nv[mt][0] & 0xffu) | ((nv[mt][1] & 0xffu) << 8);
                const uint32_t s2 = e4m3x2_to_f16x2(pair);
                const uint32_t slo2 = __byte_perm(s2, 0u, 0x1010), shi2 = __byte_perm(s2, 0u, 0x3232);
                l0 = hmul2_u32(l0, slo2); l1 = hmul2_u32(l1, slo2); l2 = hmul2_u32(l2, slo2); l3 = hmul2_u32(l3, slo2);
                h0 = hmul2_u32(h0, shi2); h1 = hmul2_u32(h1, shi2); h2 = hmul2_u32(h2, shi2); h3 = hmul2_u32(h3, shi2);
              }
              A[mt][0][0] = l0; A[mt][0][1] = h0; A[mt][0][2] = l1; A[mt][0][3] = h1;
              A[mt][1][0] = l2; A[mt][1][1] = h2; A[mt][1][2] = l3; A[mt][1][3] = h3;
            }
          }
          if constexpr (F == kINT4) {
            // constant part of this 128-wide group's offset products, per column
            if ((b & 3) == 0) {
              const int grp = (ch * KC + b * 32) / 128;
#pragma unroll
              for (int q = 0; q < NQ; ++q) {
                if (kGuard && q >= ng_act) break;
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) gbias[q][hc] = __ldg(a.xbias + gb_off[q][hc] + grp);
              }
            }
          }
          // activation fragment: box b/2, granule (b&1)*4 + c of row q*8 + sigma(g)
          const uint32_t xa = ((b & 1) ? xa1 : xa0) + (uint32_t)(b >> 1) * (XCOLS * kLine);
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            if (kGuard && q >= ng_act) break;
            const uint4 xv = lds128(xa + q * 8 * kLine);
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
              if constexpr (F == kMXFP4) {
                float t4[4];
                mma_f16_z(t4, A[mt][0][0], A[mt][0][1], A[mt][0][2], A[mt][0][3], xv.x, xv.y);
                mma_f16(t4, A[mt][1][0], A[mt][1][1], A[mt][1][2], A[mt][1][3], xv.z, xv.w);
                ffma2_scalar(acc[q][mt][0], acc[q][mt][1], t4[0], t4[1], scb[mt][0]);
                ffma2_scalar(acc[q][mt][2], acc[q][mt][3], t4[2], t4[3], scb[mt][1]);
              } else if constexpr (F == kINT4) {
                if ((b & 3) == 0)
                  mma_f16_z(tmp[q][mt], A[mt][0][0], A[mt][0][1], A[mt][0][2], A[mt][0][3], xv.x, xv.y);
                else
                  mma_f16(tmp[q][mt], A[mt][0][0], A[mt][0][1], A[mt][0][2], A[mt][0][3], xv.x, xv.y);
                mma_f16(tmp[q][mt], A[mt][1][0], A[mt][1][1], A[mt][1][2], A[mt][1][3], xv.z, xv.w);
              } else if constexpr (F == kNVFP4) {
                mma_f16(acc[q][mt], A[mt][0][0], A[mt][0][1], A[mt][0][2], A[mt][0][3], xv.x, xv.y);
                mma_f16(acc[q][mt], A[mt][1][0], A[mt][1][1], A[mt][1][2], A[mt][1][3], xv.z, xv.w);
              } else {
                mma_bf16(acc[q][mt], A[mt][0][0], A[mt][0][1], A[mt][0][2], A[mt][0][3], xv.x, xv.y);
                mma_bf16(acc[q][mt], A[mt][1][0], A[mt][1][1], A[mt][1][2], A[mt][1][3], xv.z, xv.w);
              }
            }
          }
          if constexpr (F == kINT4) {
            // end of a 128-wide scale group (or of the row): scale and accumulate
            if ((b & 3) == 3 || b == nblk - 1) {
              const int gi = b >> 2;  // group inside the chunk: bf16 half gi of the chunk word
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                const uint32_t wlo = __shfl_sync(0xffffffffu, sv[0], (lane & ~3) | (2 * mt));
                const uint32_t whi = __shfl_sync(0xffffffffu, sv[0], (lane & ~3) | (2 * mt + 1));
                const float s_lo = __uint_as_float(gi ? (wlo & 0xffff0000u) : (wlo << 16));
                const float s_hi = __uint_as_float(gi ? (whi & 0xffff0000u) : (whi << 16));
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                  if (kGuard && q >= ng_act) break;
                  const float t0 = tmp[q][mt][0] - gbias[q][0], t1 = tmp[q][mt][1] - gbias[q][1];
                  const float t2 = tmp[q][mt][2] - gbias[q][0], t3 = tmp[q][mt][3] - gbias[q][1];
                  ffma2_scalar(acc[q][mt][0], acc[q][mt][1], t0, t1, s_lo);
                  ffma2_scalar(acc[q][mt][2], acc[q][mt][3], t2, t3, s_hi);
                }
              }
            }
          }
        };
        using IFull = std::integral_constant<int, NG>;
        using IOne = std::integral_constant<int, 1>;
        if (nblk == KC / 32) {
          // full chunk: straight-line code, every block and column group static
          if (ng_act >= NG) {
#pragma unroll
            for (int b = 0; b < KC / 32; ++b) block(b, IFull{}, std::false_type{});
          } else if (NG > 1 && ng_act == 1) {
#pragma unroll
            for (int b = 0; b < KC / 32; ++b) block(b, IOne{}, std::false_type{});
          } else {
#pragma unroll
            for (int b = 0; b < KC / 32; ++b) block(b, IFull{}, std::true_type{});
          }
        } else {
#pragma unroll
          for (int b = 0; b < KC / 32; ++b) {
            if (b >= nblk) break;
            block(b, IFull{}, std::true_type{});
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      rc.next();
    }
    if (*s_abort) break;
    // ------------------------------------------------- split K: slice sums
    if constexpr (kSplit && NG == 1) {
      if (S > 1) {
        if (!(active && ncols > 0)) continue;
        constexpr int kPartF = kMT * 4;  // this thread's accumulators
        const size_t thr = (size_t)(warp * 32 + lane) * 8;
        float* part0 = a.split_part + (size_t)base * S * (kConsumerWarps * 32 * 8) + thr;
        float* mine = part0 + (size_t)slice * (kConsumerWarps * 32 * 8);
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
          __stcg(reinterpret_cast<float4*>(mine) + mt, make_float4(acc[0][mt][0], acc[0][mt][1], acc[0][mt][2], acc[0][mt][3]));
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(a.split_ctr + (size_t)base * kConsumerWarps + warp, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != S - 1) continue;  // another slice's warp finishes these rows
        __threadfence();
        // every slice's partial, summed in slice order (the same sum whichever warp is last)
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(part0) + mt);
          acc[0][mt][0] = v.x; acc[0][mt][1] = v.y; acc[0][mt][2] = v.z; acc[0][mt][3] = v.w;
        }
        for (int sl = 1; sl < S; ++sl) {
          const float4* ps = reinterpret_cast<const float4*>(part0 + (size_t)sl * (kConsumerWarps * 32 * 8));
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt) {
            const float4 v = __ldcg(ps + mt);
            acc[0][mt][0] += v.x; acc[0][mt][1] += v.y; acc[0][mt][2] += v.z; acc[0][mt][3] += v.w;
          }
        }
        static_assert(kPartF <= 8, "partial slots per thread");
      }
    }
    // ---------------------------------------------------------- epilogue
    if (active && ncols > 0) {
#pragma unroll
      for (int q = 0; q < NG; ++q) {
        if (q < ng_act) {
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            const int col = c0 + q * 8 + sigma8(2 * c + hc);  // activation row inside the expert
            if (col < it.n_cols) {
              const int xrow = it.xrow0 + col;
              float f = it.gscale;
              if (F != kBF16) f = ldexpf(f, __ldg(a.xexp + xrow));
              // weight rows held by this lane: (row g, row g+8) of each m-tile (bf16: sigma(g))
              const int wr = (F == kBF16) ? sg : g;
              if (kGateUp) {
                __nv_bfloat16* o = a.out_routed + (int64_t)xrow * a.N + r0 + m0;
                if constexpr (kHalf) {
                  // one m-tile: rows g hold the gate, rows g+8 the up projection
                  const float gt = acc[q][0][hc] * f;
                  const float up = acc[q][0][2 + hc] * f;
                  o[wr] = __float2bfloat16_rn(gt / (1.f + expf(-gt)) * up);
                } else {
#pragma unroll
                  for (int hr = 0; hr < 2; ++hr) {
                    const float gt = acc[q][0][hr * 2 + hc] * f;
                    const float up = acc[q][kMT - 1][hr * 2 + hc] * f;
                    const float h = gt / (1.f + expf(-gt)) * up;
                    o[wr + 8 * hr] = __float2bfloat16_rn(h);
                  }
                }
              } else {
                __nv_bfloat16* o = it.shared_idx >= 0
                                       ? a.out_shared + ((int64_t)it.shared_idx * a.T + col) * a.N
                                       : a.out_routed + (int64_t)xrow * a.N;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                  for (int hr = 0; hr < 2; ++hr)
                    o[r0 + m0 + mt * 16 + wr + 8 * hr] = __float2bfloat16_rn(acc[q][mt][hr * 2 + hc] * f);
              }
            }
          }
        }
      }
    }
  }
  if constexpr (Tr::blk != 0) {
    // every consumer warp is done with tensor memory before warp 0 frees it
    tc::fence_before_sync();
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    if (warp == 0) {
      tc::fence_after_sync();
      tc::tmem_dealloc(*s_tmem, (uint32_t)a.tmem_alloc);
    }
  }
}

// ------------------------------------------------------------------ host side
template <int F, int NG, bool GU, int MINB, bool HALF, bool SPLIT = false>
static cudaError_t launch_one(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto kern = ffn_stream_kernel<F, NG, GU, MINB, HALF, SPLIT>;
  {
    cudaError_t err = set_dyn_smem_once<ffn_stream_kernel<F, NG, GU, MINB, HALF, SPLIT>>(smem);
    if (err != cudaSuccess) return err;
  }
  if (a.tmem_alloc > 0) {
    // tcgen05.alloc waits while the SM's 512 columns are taken: never let the
    // blocks that can share an SM ask for more than that together.
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm * a.tmem_alloc > 512) return cudaErrorInvalidConfiguration;
  }
  ProfScope prof(GU ? "ffn_stage1_gate_up" : "ffn_stage2_down", st);
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, a);
}

template <int F, bool GU>
static cudaError_t dispatch_ng(const FfnArgs& a, int ng, int minb, bool half, int grid, size_t smem,
                               cudaStream_t st) {
  if (a.split > 1) {  // split K: one column group
    if (half) {
      if (minb == 3) return launch_one<F, 1, GU, 3, true, true>(a, grid, smem, st);
      return launch_one<F, 1, GU, 2, true, true>(a, grid, smem, st);
    }
    if (minb == 3) return launch_one<F, 1, GU, 3, false, true>(a, grid, smem, st);
    if (minb == 2) return launch_one<F, 1, GU, 2, false, true>(a, grid, smem, st);
    return launch_one<F, 1, GU, 1, false, true>(a, grid, smem, st);
  }
  if (half) {  // one column group, two or three blocks per SM
    if (minb == 3) return launch_one<F, 1, GU, 3, true>(a, grid, smem, st);
    return launch_one<F, 1, GU, 2, true>(a, grid, smem, st);
  }
  if (minb == 3) return launch_one<F, 1, GU, 3, false>(a, grid, smem, st);
  if (minb == 2) {
    switch (ng) {
      case 1: return launch_one<F, 1, GU, 2, false>(a, grid, smem, st);
      default: return launch_one<F, 2, GU, 2, false>(a, grid, smem, st);
    }
  }
  switch (ng) {
    case 1: return launch_one<F, 1, GU, 1, false>(a, grid, smem, st);
    case 2: return launch_one<F, 2, GU, 1, false>(a, grid, smem, st);
    default: return launch_one<F, 4, GU, 1, false>(a, grid, smem, st);
  }
}

static int fmt_kc(int F) { return F == kBF16 ? 64 : 256; }
static int fmt_srow(int F, int K) {
  switch (F) {
    case kMXFP4: return K / 32;
    case kNVFP4: return K / 16;
    case kINT4: return (K / 128) * 2;
    default: return 0;
  }
}

// Shared memory plan of one stage kernel: the header, then a ring of stages
// (weights + activations).  Block scales travel through the same ring, one
// item's scales in n_sslots stages, so no buffer is set aside for them.
// Returns false when fewer than two stages fit.
static bool plan_smem(int F, int ng, int K, int E, int n_shared, int smem_max, bool half, FfnArgs& a,
                      size_t& total) {
  const int hdr = stream_hdr_bytes(E, n_shared);
  const int wrows = half ? kRowsPerStage / 2 : kRowsPerStage;  // weight rows per stage
  const int stage = wrows * kLine + ((fmt_kc(F) * 2) / kLine) * ng * 8 * kLine;
  const int usable = smem_max - 1024;  // room for the runtime 1024-byte alignment
  int ns = (usable - hdr) / stage;
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < 2) return false;
  a.n_stages = ns;
  a.n_sslots = 0;
  const int srow = fmt_srow(F, K);
  if (srow > 0) {
    // each of the 8 consumer warps owns 32 scale rows (16 with half items);
    // split them over 1, 2, 4 or 8 stages
    const int per_warp = half ? 16 : 32;
    int n = 1;
    while (n < kConsumerWarps && (kConsumerWarps / n) * per_warp * srow > stage) n *= 2;
    if ((kConsumerWarps / n) * per_warp * srow > stage) return false;
    a.n_sslots = n;
  }
  total = (size_t)1024 + hdr + (size_t)ns * stage;
  return true;
}

// TMEM columns for one weight row's block scales: whole 32-bit words, a
// multiple of 4 (the copy-in stores 4 at a time) and at least every column a
// K chunk reads.
static int tmem_scale_cols(int F, int K) {
  const int srow = fmt_srow(F, K);
  if (srow == 0) return 0;
  const int cpc = F == kMXFP4 ? 2 : (F == kNVFP4 ? 4 : 1);
  int cols = (((srow + 3) / 4) + 3) & ~3;
  const int need = ceil_div(K, fmt_kc(F)) * cpc;
  if (cols < need) cols = (need + 3) & ~3;
  return cols;
}

cudaError_t launch_ffn_stream(int F, bool gate_up, FfnArgs a, const FfnPointers& p, int T, int n_sms,
                              int smem_max, int smem_per_sm, cudaStream_t st, int* unsupported) {
  *unsupported = 0;
  // Columns per pass (NG groups of 8 activation rows) and CTAs per SM.  Two
  // CTAs of 8 consumer warps hide the decode's fixed-latency dependencies
  // better than one (measured on the gpt-oss decode batch: stage 1 at 4.2 vs
  // 3.2 TB/s).  One group of 8 columns covers almost every routed expert of a
  // decode batch that averages a few rows per expert, and leaves room for the
  // activation boxes; shared experts (T rows each) and batches that average
  // four or more rows per expert take 16 columns per pass (measured: Kimi
  // T=128 1.48 vs 1.67 ms per layer with 16 vs 8, gpt-oss T=64 350 vs 356 us
  // with 8 vs 16).  Weight boxes keep normal L2 priority: a 128-byte box row
  // of a 1440-byte weight row straddles 64-byte lines whose other half the
  // next K chunk reads, and marking them evict-first let L2 drop those halves
  // before that (DRAM reads 1.125 vs 1.042 GB per stage-1 launch; stage 1
  // 229 vs 204 us at T=64).  MOE_FFN_NG / MOE_FFN_MINB / MOE_W_L2FIRST
  // override the choices for tuning.  Batches of up to 16 tokens take one
  // group even with shared experts (Kimi-shaped layer, T=16: 372 vs 384 us
  // per layer; T=32: 564 vs 559 us, so two groups from there).
  int ng = (T <= 16 || (a.n_shared == 0 && (int64_t)T * a.k < 4LL * a.E)) ? 1 : 2;
  // With one column group a block fits in a third of an SM (two stages of
  // 36 KB, 72 registers a thread): 24 consumer warps per SM hide more of the
  // decode's dependency latency than 16 (gpt-oss T=64: stage 1 at 0.77 vs 0.74
  // of the HBM copy peak; T=8 121 vs 128 us per layer).
  int minb = ng == 1 ? 3 : 2;
  if (const char* e = getenv("MOE_FFN_NG")) ng = atoi(e);
  if (const char* e = getenv("MOE_FFN_MINB")) minb = atoi(e);
  if (ng != 1 && ng != 2 && ng != 4) ng = 2;
  if (const char* e = getenv("MOE_W_L2FIRST")) a.w_l2_first = atoi(e);
  if (minb == 2 && ng > 2) ng = 2;
  if (minb == 3 && ng != 1) minb = 2;
  // Half items (128 rows of W_down) in stage 2 when full items would fill
  // fewer than half of the block slots: twice the blocks stream the same
  // bytes (gpt-oss T=1: stage 2 19.0 vs 23.0 us).  Measured not to pay in
  // stage 1 (64 + 64-row items: 24.3 vs 23.0 us) nor with long K rows (Kimi
  // T=1, 28 chunks per item either way: 133 vs 126 us per layer), where each
  // block's chain of stage round trips, not its bytes, sets the time.
  // MOE_FFN_HALF=0/1 overrides (either stage).
  bool half;
  {
    const long full_items = (long)(a.n_shared + (a.E < T * a.k ? a.E : T * a.k)) * ceil_div(a.N, gate_up ? 128 : 256);
    half = !gate_up && ng == 1 && minb >= 2 && 2 * full_items < (long)n_sms * minb;
    if (const char* e = getenv("MOE_FFN_HALF")) half = atoi(e) != 0 && ng == 1 && minb >= 2;
  }
  size_t smem = 0;
  bool ok = false;
  if (minb == 3) ok = plan_smem(F, ng, a.K, a.E, a.n_shared, smem_per_sm / 3 - 1024, half, a, smem);
  if (!ok && minb == 3) minb = 2;
  if (minb == 2) ok = plan_smem(F, ng, a.K, a.E, a.n_shared, smem_per_sm / 2 - 1024, half, a, smem);
  if (!ok) {
    minb = 1;
    half = false;
    ok = plan_smem(F, ng, a.K, a.E, a.n_shared, smem_max, false, a, smem);
  }
  if (!ok) {
    *unsupported = 1;
    return cudaSuccess;
  }
  // TMEM for the block scales: 2 x tmem_cols columns (two warps per lane
  // quarter), at most 256 per block so that two co-resident blocks never wait
  // for each other's columns (launch_one checks the occupancy).
  a.tmem_cols = tmem_scale_cols(F, a.K);
  a.tmem_alloc = 0;
  if (a.tmem_cols > 0) {
    int alloc = 32;
    while (alloc < 2 * a.tmem_cols) alloc *= 2;
    if (alloc > 256) {
      *unsupported = 1;  // more than 512 scale bytes per weight row
      return cudaSuccess;
    }
    if (minb == 3 && 3 * alloc > 512) {
      // three blocks per SM would not all get their columns: two per SM
      minb = 2;
      if (!plan_smem(F, ng, a.K, a.E, a.n_shared, smem_per_sm / 2 - 1024, half, a, smem)) {
        *unsupported = 1;
        return cudaSuccess;
      }
    }
    a.tmem_alloc = alloc;
  }
  // tensor maps (MOE_W_PROMO=0|64|128|256: the L2 promotion of the weight
  // boxes, for measuring the DRAM traffic of rows whose 128-byte boxes do
  // not start on 128-byte lines)
  int w_promo = 256;
  if (const char* e = getenv("MOE_W_PROMO")) w_promo = atoi(e);
  const uint64_t row_bytes = (F == kBF16) ? (uint64_t)a.K * 2 : (uint64_t)a.K / 2;
  const uint64_t wrows = gate_up ? 2 * (uint64_t)a.N : (uint64_t)a.N;
  const uint32_t box_rows = (gate_up && half) ? 64u : (uint32_t)kBoxRows;  // rows per weight box
  {
    const uint64_t dims[3] = {row_bytes, wrows, (uint64_t)a.n_phys};
    const uint64_t strides[2] = {row_bytes, (uint64_t)p.stride_w};
    const uint32_t box[3] = {kLine, box_rows, 1};
    if (!encode_tmap_u8(&a.tm_w, p.w, 3, dims, strides, box, true, w_promo)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  }
  if (a.n_shared > 0) {
    const uint64_t dims[3] = {row_bytes, wrows, (uint64_t)a.n_shared};
    const uint64_t strides[2] = {row_bytes, (uint64_t)p.stride_w_sh};
    const uint32_t box[3] = {kLine, box_rows, 1};
    if (!encode_tmap_u8(&a.tm_wsh, p.w_sh, 3, dims, strides, box, true, w_promo)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  } else {
    a.tm_wsh = a.tm_w;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.K * 2, (uint64_t)p.rows_total};
    const uint64_t strides[1] = {(uint64_t)a.K * 2};
    const uint32_t box[2] = {kLine, (uint32_t)(ng * 8)};
    if (!encode_tmap_u8(&a.tm_x, p.x, 2, dims, strides, box, true)) {
      *unsupported = 1;
      return cudaSuccess;
    }
  }
  const int rows_per_item = gate_up ? (half ? 64 : 128) : (half ? 128 : 256);
  const int ntile = ceil_div(a.N, rows_per_item);
  const long max_items = (long)(a.n_shared + (a.E < T * a.k ? a.E : T * a.k)) * ntile;
  const long slots = (long)n_sms * minb;
  // Split K (off by default; MOE_FFN_SPLIT=S asks for S slices): each block
  // decodes a slice of an item's K chunks, for batches of a few tokens whose
  // items would leave most block slots idle; one pass per item (T <= 8)
  // keeps the item count the bound computed here.  Measured on B200 it does
  // not pay: the gpt-oss-shaped layer at T = 1 with 4 slices takes 54.8 vs
  // 53.5 us per layer, because a block's time there is set by the launch
  // ramp, its setup, the first burst of loads all blocks issue at once and
  // the epilogue, not by its decode work (timestamps per block: stage 1 takes
  // ~16 us after its predecessor ends either way), and every slice re-reads
  // the item's block scales.
  int split = 1;
  if (ng == 1 && a.split_cap > 0 && T <= 8 && max_items > 0) {
    const int nch = ceil_div(a.K, fmt_kc(F));
    if (const char* e = getenv("MOE_FFN_SPLIT")) {
      const int v = atoi(e);
      if (v >= 1 && v <= 8 && max_items * v <= a.split_cap && nch >= v) split = v;
    }
  }
  a.split = split;
  const long work = max_items * split;
  int grid = (int)(work < slots ? work : slots);
  if (grid < 1) return cudaSuccess;
  switch (F) {
    case kBF16: return gate_up ? dispatch_ng<kBF16, true>(a, ng, minb, half, grid, smem, st) : dispatch_ng<kBF16, false>(a, ng, minb, half, grid, smem, st);
    case kMXFP4: return gate_up ? dispatch_ng<kMXFP4, true>(a, ng, minb, half, grid, smem, st) : dispatch_ng<kMXFP4, false>(a, ng, minb, half, grid, smem, st);
    case kNVFP4: return gate_up ? dispatch_ng<kNVFP4, true>(a, ng, minb, half, grid, smem, st) : dispatch_ng<kNVFP4, false>(a, ng, minb, half, grid, smem, st);
    default: return gate_up ? dispatch_ng<kINT4, true>(a, ng, minb, half, grid, smem, st) : dispatch_ng<kINT4, false>(a, ng, minb, half, grid, smem, st);
  }
}

}  // namespace moe
