/*
 * moe.h - C ABI of a B200 (sm_100a) library for the forward pass of one sparse
 * mixture-of-experts (MoE) layer:
 *
 *   router product -> top-k experts with renormalised softmax gates ->
 *   stable per-expert permutation -> grouped SwiGLU expert FFN over bf16,
 *   MXFP4, NVFP4 or INT4 group-128 weights (decoded inside the kernels) ->
 *   weighted combine back to token order (+ shared experts),
 *
 * plus an HBM expert cache filled from a pinned host-memory expert bank.
 *
 * What the pages define, and where:
 *  - "Each MoE layer replaces the dense feed-forward block with many smaller
 *    expert blocks and a router that picks a few of them per token"; attention,
 *    embeddings and the router stay dense ("Mixture of experts VRAM: total vs
 *    active parameters", section "How current MoE models route each token").
 *  - Top-k counts and shared experts (same page and section: 4 of 128 for
 *    gpt-oss-120b; Kimi-K2.6 8 of 384 plus one shared expert; Llama 4 Maverick
 *    "Each token is sent to the shared expert and also to one of the 128 routed
 *    experts").
 *  - Experts have gate, up and down projections (FloE verdict page, JSON field
 *    referee_report.summary).
 *  - 4-bit experts: FP4 (gpt-oss, DeepSeek-V4-Flash) and INT4 (Kimi) (page
 *    "Mixture of experts VRAM", same section); MXFP4 and native-INT4 exports
 *    ("Understanding MoE Inference Costs on Galactus", August table).
 *  - Prefill groups the tokens that select the same expert so one weight read
 *    serves many activations (Galactus page, section "Prompt processing is a
 *    different phase"); decode reads each token's active experts (page
 *    "Mixture of experts VRAM", section "What active parameters change").
 *  - Expert paging through stable logical slots whose physical residency moves
 *    underneath ("Running MoE LLMs on a single GPU: what expert offloading
 *    actually costs", section "Inside expert paging"); an LRU expert cache
 *    (related-papers feed, locality-trained routers abstract).
 *
 * Conventions (all entry points):
 *  - Ownership: the caller owns every device buffer and the stream.  No entry
 *    point of the layer path allocates memory; scratch comes from the caller's
 *    `workspace` (size from moe_workspace_size).  The workspace needs no
 *    initialisation and holds nothing between calls: the counters a call uses
 *    are zeroed by that call's own kernels.  The expert cache owns what
 *    moe_cache_init allocates.
 *  - On-chip resources: while they run, the blocks of the 4-bit streaming FFN
 *    kernels each hold up to 256 columns of an SM's tensor memory (TMEM) for
 *    their block scales; a kernel of another library that holds all 512
 *    columns of an SM delays them until it finishes.
 *  - Execution: every compute call enqueues work on `stream` and returns; host
 *    argument checks return synchronously (MOE_ERR_INVALID_ARG /
 *    MOE_ERR_UNSUPPORTED) before anything is enqueued.  Launch failures return
 *    MOE_ERR_CUDA.  Errors found by the kernels (an expert index out of range, a
 *    bounded wait that ran out) are written to a sticky device status word that
 *    moe_get_last_error() reads (it synchronises the device).
 *  - Pointers are device pointers unless marked "host", 16-byte aligned.
 *  - Layouts are row-major.  Expert matrices are K-major [E][N][K]: W13 has
 *    2*d_ff rows (rows [0, d_ff) gate, rows [d_ff, 2*d_ff) up) of d_model
 *    columns; W2 has d_model rows of d_ff columns.  4-bit codes are packed two
 *    per byte, even K in the low nibble.  Block scales are [E][N][K/blk]:
 *      MXFP4 : E2M1 codes, one E8M0 byte per 32 K            (value = e2m1 * 2^(s-127))
 *      NVFP4 : E2M1 codes, one E4M3 byte per 16 K, fp32 per-expert global scale
 *      INT4  : two's complement codes, one bf16 scale per 128 K
 *      BF16  : plain bf16 values, no scales.
 *  - Shapes: d_model and d_ff must be multiples of 32 (of 128 for INT4);
 *    1 <= top_k <= min(n_experts, 32); n_experts <= 1024; T >= 0 (T = 0 is a
 *    no-op that returns MOE_OK).  The 4-bit streaming FFN keeps at most 512
 *    scale bytes per weight row in tensor memory: a reduction length beyond
 *    16384 (MXFP4), 8192 (NVFP4) or 32768 (INT4) returns MOE_ERR_UNSUPPORTED.
 *  - Numerics: activations bf16, products accumulated in fp32.  The 4-bit paths
 *    feed the tensor cores fp16 operands: E2M1 codes convert to fp16 exactly,
 *    and each activation row is scaled by a power of two so that it fits fp16
 *    (exact for every value of magnitude at least 2^-31 times its row's
 *    largest); the power of two is undone on the fp32 accumulator.  INT4 codes
 *    enter as the exact fp16 integers 1024 + 16^j (q + 8) against activations
 *    pre-divided by 16 where j = 1, and the constant part of each 128-group
 *    is subtracted from the fp32 group sum before the group scale.
 *  - Thread safety: calls on different streams with different workspaces may
 *    run concurrently; an expert cache object is not thread-safe.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,     /* null pointer, bad shape, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,     /* valid but outside what the library handles */
  MOE_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed */
  MOE_ERR_OOM = 4,             /* cache allocation failed */
  MOE_ERR_CACHE_PINNED_FULL = 5, /* every slot of a layer is protected */
  MOE_ERR_TIMEOUT = 6,         /* a bounded device-side wait gave up */
  MOE_ERR_INJECTED = 7,        /* a host-side fault injection fired */
  MOE_ERR_WORKSPACE = 8,       /* workspace smaller than moe_workspace_size */
  MOE_ERR_DEVICE_INDEX = 9     /* a kernel saw an expert/slot index out of range */
} moe_status;

typedef enum { MOE_W_BF16 = 0, MOE_W_MXFP4 = 1, MOE_W_NVFP4 = 2, MOE_W_INT4_G128 = 3 } moe_wdtype;

typedef struct {
  int32_t T;           /* tokens in this call */
  int32_t d_model;     /* hidden size d */
  int32_t n_experts;   /* routed experts E */
  int32_t top_k;       /* experts per token k */
  int32_t d_ff;        /* expert FFN width */
  int32_t n_shared;    /* shared experts, each applied to every token with weight 1 */
  int32_t wdtype;      /* moe_wdtype of the expert weights */
  int32_t router_fp32; /* 0: router weights bf16 [E][d]; 1: fp32 [E][d] */
} moe_layer_desc;

/* Expert weights of one layer (routed or shared).  Expert e's tensors start at
 * base + p * stride, where p = slot_map ? slot_map[e] : e (a stride of 0 means
 * tightly packed).  Strides are in bytes and must be multiples of 16.  g13/g2
 * (NVFP4 only) are indexed by the logical expert e.  With a slot map, an entry
 * of -1 means "not resident": that expert is skipped and its rows of y_perm
 * are left unwritten (an expert cache serving a need set in waves fills them
 * in later calls); an entry >= n_physical sets MOE_ERR_DEVICE_INDEX. */
typedef struct {
  const void* w13;     /* [.][2*d_ff][d] values or packed codes */
  const void* s13;     /* [.][2*d_ff][d/blk] block scales, NULL for BF16 */
  const void* w2;      /* [.][d][d_ff] */
  const void* s2;      /* [.][d][d_ff/blk] */
  const float* g13;    /* [E] NVFP4 global scales of W13, else NULL */
  const float* g2;     /* [E] NVFP4 global scales of W2, else NULL */
  int64_t stride_w13, stride_s13, stride_w2, stride_s2;
  const int32_t* slot_map; /* device [E] logical -> physical expert, or NULL */
  int32_t n_physical;      /* experts the bases hold (0: n_experts, or n_shared for shared) */
} moe_weights;

/* Byte offsets of the routing results inside a moe_layer_forward workspace. */
typedef struct {
  size_t topk_idx;   /* int32 [T][k] */
  size_t topk_w;     /* fp32  [T][k] */
  size_t offsets;    /* int32 [E+1] */
  size_t row_token;  /* int32 [T*k] */
  size_t inv;        /* int32 [T*k] */
  size_t total;      /* = moe_workspace_size */
} moe_workspace_layout;

/* Depth of the fp32 summation tree each router logit goes through (used to
 * bound its rounding error): 8*ceil(d/2048) + 12 additions. */
#define MOE_ROUTER_SUM_DEPTH(d) (8 * (((d) + 2047) / 2048) + 12)

/* Scratch bytes moe_layer_forward needs for `desc` (also enough for
 * moe_route_topk and moe_grouped_ffn).  No counterpart in the pages: the
 * caller-owned scratch of this library's calls. */
moe_status moe_workspace_size(const moe_layer_desc* desc, size_t* bytes);
moe_status moe_workspace_layout_of(const moe_layer_desc* desc, moe_workspace_layout* out);

/* Router and top-k ("Mixture of experts VRAM: total vs active parameters",
 * section "How current MoE models route each token": a dense router picks k
 * experts per token).  logits[t][e] = sum_i x[t][i]*Wr[e][i] (+ logit_bias[e]),
 * fp32 accumulation; per token the k largest logits in descending order, the
 * lower expert index winning ties; topk_w = softmax over the selected logits
 * (equal to the softmax over all E renormalised over the selection).
 * x: bf16 [T][d]; w_router: bf16 or fp32 [E][d]; logit_bias: fp32 [E] or NULL.
 * Outputs topk_idx int32 [T][k], topk_w fp32 [T][k].  Needs `workspace` for
 * the fp32 logits (T*E*4 bytes; moe_route_topk_noalloc keeps them in the
 * library instead). */
moe_status moe_route_topk(const moe_layer_desc* desc, const void* x, const void* w_router,
                          const float* logit_bias, int32_t* topk_idx, float* topk_w,
                          void* workspace, size_t ws_bytes, void* stream);

/* moe_route_topk for callers that cannot allocate device memory (no
 * counterpart in the paper: an interface convenience of this library).
 * Same inputs, outputs and arithmetic as moe_route_topk, but the fp32 logits
 * scratch is a fixed device array inside the library instead of a caller
 * workspace: for plugins whose host framework owns every device allocation,
 * or runtimes that fix their device memory at start-up.  Limit: T * n_experts
 * <= 262144 (1 MiB, held on every GPU that loads the library until exit);
 * larger calls return MOE_ERR_WORKSPACE before enqueueing anything.  The
 * first call on a device looks up the array's device address (make it before
 * any stream capture); a call that finds another context current on that
 * device (after cudaDeviceReset, say) looks it up again.  Calls share the
 * array: calls that overlap on the GPU race.  Nothing is allocated. */
moe_status moe_route_topk_noalloc(const moe_layer_desc* desc, const void* x, const void* w_router,
                                  const float* logit_bias, int32_t* topk_idx, float* topk_w, void* stream);

/* Stable counting sort of the T*k (token, slot) pairs by expert (Galactus
 * page, section "Prompt processing is a different phase": the tokens that
 * select one expert are grouped so one weight read serves them all).
 * offsets int32 [E+1] (exclusive prefix sum of per-expert counts),
 * row_token int32 [T*k] (token of each grouped row; rows of one expert are in
 * ascending token order), inv int32 [T*k] (row of pair t*k+j).  With x
 * (bf16 [T][d]) non-NULL the activation rows are also gathered into expert
 * order: x_perm bf16 [T*k][d], x_perm[r] = x[row_token[r]] (x NULL: no
 * gather, x_perm ignored; moe_grouped_ffn gathers by itself from x).  An
 * index outside [0, E) sets MOE_ERR_DEVICE_INDEX in the device status word
 * and the pair is dropped (its gathered row, if any, is zero). */
moe_status moe_permute(const moe_layer_desc* desc, const int32_t* topk_idx, const void* x, int32_t* offsets,
                       int32_t* row_token, int32_t* inv, void* x_perm, void* stream);

/* Grouped SwiGLU expert FFN (gate, up and down projections: FloE verdict
 * page, JSON field referee_report.summary; grouping: Galactus page, section
 * "Prompt processing is a different phase").  For every routed row r of expert e (rows
 * [offsets[e], offsets[e+1])) with token t = row_token[r]:
 *   y_perm[r] = W2_e (silu(W_gate,e x_t) * (W_up,e x_t)),
 * and for every shared expert s and token t: y_shared[s][t] likewise.
 * x: bf16 [T][d]; y_perm bf16 [T*k][d]; y_shared bf16 [n_shared][T][d] (NULL
 * when n_shared = 0).  The intermediate h is rounded to bf16.  Each routed
 * expert's weights are read from HBM once per call when it has <= 32 rows. */
moe_status moe_grouped_ffn(const moe_layer_desc* desc, const moe_weights* routed,
                           const moe_weights* shared, const int32_t* offsets,
                           const int32_t* row_token, const void* x, void* y_perm, void* y_shared,
                           void* workspace, size_t ws_bytes, void* stream);

/* Weighted combine ("Mixture of experts VRAM", section "How current MoE
 * models route each token": routed experts weighted by the router, the shared
 * expert on every token):
 * out[t] = sum_{j<k} topk_w[t][j] * y_perm[inv[t*k+j]]
 *                            + sum_s y_shared[s][t]   (fp32 sum in that order),
 * out bf16 [T][d]. */
moe_status moe_combine(const moe_layer_desc* desc, const void* y_perm, const int32_t* inv,
                       const float* topk_w, const void* y_shared, void* out, void* stream);

/* The whole layer (the four calls above, in the pages' order):
 * route_topk -> permute -> grouped_ffn -> combine, all on
 * `stream`, scratch in `workspace` (layout: moe_workspace_layout_of). */
moe_status moe_layer_forward(const moe_layer_desc* desc, const void* x, const void* w_router,
                             const float* logit_bias, const moe_weights* routed,
                             const moe_weights* shared, void* out, void* workspace,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Expert cache: per-layer LRU over HBM slots, filled from a pinned host bank.
 * Policy (per layer, `slots_per_layer` slots): lookup walks its experts in
 * ascending id, in waves of at most slots_per_layer; a resident expert (copied
 * by an earlier miss or prefetch) is a hit; a miss takes the lowest free slot,
 * else evicts the least recently used expert not in the current wave; every
 * access makes the expert most recently used.  Prefetch inserts the listed
 * non-resident experts (ascending, at most slots_per_layer) the same way,
 * never evicting another expert of the same call.  Copies run with
 * cudaMemcpyAsync on the cache's own copy stream; a slot is overwritten only
 * after the compute work that last read it (recorded by moe_cache_release).
 * ---------------------------------------------------------------------- */
typedef struct moe_cache moe_cache;

typedef struct {
  int32_t n_layers;
  int32_t n_experts;       /* experts per layer */
  int32_t slots_per_layer; /* HBM slots per layer */
  int64_t expert_bytes;    /* bytes of one expert blob (multiple of 16) */
  void* host_bank;         /* host: pinned [n_layers][n_experts][expert_bytes], or NULL to
                              allocate (cudaHostAlloc) */
  int32_t device;          /* CUDA device of the slots; < 0: policy only (no memory, no copies, no
                              CUDA calls; lookup accepts a NULL slot map) - the replacement
                              policy and counters alone, for replaying traces */
} moe_cache_desc;

typedef struct {
  int64_t lookups, hits, misses, evictions, prefetch_issued, prefetch_used;
  int64_t bytes_h2d;
  double copy_ms; /* sum of completed copy durations (events) */
} moe_cache_stats_t;

/* Allocates the HBM slots (slots_per_layer per layer), the pinned bank
 * (unless given), the copy stream and events ("Running MoE LLMs on a single
 * GPU: what expert offloading actually costs", section "Inside expert
 * paging": stable logical slots, physical residency below them). */
moe_status moe_cache_init(moe_cache** cache, const moe_cache_desc* desc);
/* Host pointer to layer `layer`, expert `e` in the bank (to fill it). */
void* moe_cache_host_expert(moe_cache* cache, int32_t layer, int32_t e);
/* Device base of the slot pool of `layer` (slot s at base + s*expert_bytes). */
void* moe_cache_slot_base(moe_cache* cache, int32_t layer);
/* Start copies of the listed experts of `layer` (host list) on the copy
 * stream (FloE verdict page, referee_report.summary: prefetch from the
 * current hidden state with asynchronous transfer). */
moe_status moe_cache_prefetch(moe_cache* cache, int32_t layer, const int32_t* experts /*host*/,
                              int32_t n);
/* (Expert paging, same page and section; LRU: related-papers feed.)
 * Make `experts` (host list) of `layer` resident, write the layer's logical ->
 * slot map (int32 [n_experts], -1 = absent) to slot_map_dev on `compute`
 * stream, and make `compute` wait for the copies it needs.  At most
 * slots_per_layer experts are resident at once: with a longer list the map
 * reflects the last wave, so callers serve such a need set one wave at a time
 * (lookup, compute, release per wave).  n_experts <= 1024. */
moe_status moe_cache_lookup(moe_cache* cache, int32_t layer, const int32_t* experts /*host*/,
                            int32_t n, int32_t* slot_map_dev, void* compute_stream);
/* Record that the work enqueued so far on `compute` finishes reading `layer`'s slots. */
moe_status moe_cache_release(moe_cache* cache, int32_t layer, void* compute_stream);
/* Host copy of the current slot map of `layer` (int32 [n_experts]). */
moe_status moe_cache_slot_map(const moe_cache* cache, int32_t layer, int32_t* out /*host*/);
/* Counters since init: lookups, hits, misses, evictions, prefetches issued
 * and used, bytes copied, summed copy time (the hit rate and H2D rate the
 * offloading pages report; "Running MoE LLMs on a single GPU", section "Inside
 * expert paging"). */
moe_status moe_cache_stats(moe_cache* cache, moe_cache_stats_t* out);
/* Waits for the cache's copies, frees what moe_cache_init allocated. */
moe_status moe_cache_destroy(moe_cache* cache);

/* ------------------------------------------------------------------------
 * Per-kernel device timing.  While enabled, each kernel launch of the
 * library is bracketed by two CUDA events on the stream it runs on (adds two
 * event records per launch).  moe_profile_collect waits for the recorded
 * events, writes up to `cap` entries (one per kernel name: launches and total
 * milliseconds), sets *n_out to the number of names, and clears the record.
 * Not part of the paper's method: measurement support only.
 * ---------------------------------------------------------------------- */
typedef struct {
  char name[32];
  int64_t launches;
  double total_ms;
} moe_profile_entry;
moe_status moe_profile_enable(int on);
moe_status moe_profile_collect(moe_profile_entry* out, int32_t cap, int32_t* n_out);

/* Diagnostic, no counterpart in the pages: launches one CTA that waits, with
 * the bounded wait every pipelined kernel here uses, on an mbarrier phase that
 * nothing completes.  After `limit_ns` (<= 10 s) the wait gives up, records
 * MOE_ERR_TIMEOUT in the device status word, writes 1 to *finished (device
 * int32) and the kernel returns: the failure path of a stuck pipeline,
 * exercised without hanging or faulting the GPU. */
moe_status moe_diag_wait_timeout(uint64_t limit_ns, int32_t* finished, void* stream);

const char* moe_status_string(moe_status s);
/* Synchronises the current device, returns and clears the device status word. */
moe_status moe_get_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
