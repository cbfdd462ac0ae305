/*
 * moe.h -- C ABI of a single-GPU Mixture-of-Experts layer forward for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (jsqmd.com, "第11章 MoE模型推理", 11.1.1 "稀疏激活原理"):
 *
 *     y = sum_{i in TopK} g_i(x) * E_i(x)
 *
 * runs as five steps, each exposed as its own call and chained by
 * moe_layer_forward:
 *   moe_route        router logits, scoring, top-k selection, gate weights
 *   moe_permute      expert histogram, prefix scan, stable row permutation
 *                    and gather of token rows into expert-contiguous rows
 *   moe_grouped_ffn  every expert's FFN over its rows as one grouped GEMM
 *   moe_combine      gate-weighted sum back into token order
 *
 * Around them: moe_reroute (over-capacity re-routing between two
 * permutations), moe_update_sel_bias (sliding-window selection-bias update),
 * moe_quantize_rows_e4m3 (the W8A8 activation quantiser on its own),
 * moe_split_rows_e4m3 (the two-term activation codes of E4M3-weight layers),
 * moe_permute_static (moe_permute without a workspace), and the workspace /
 * status helpers.
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers, row-major, owned by the caller.
 *    The library never allocates device or host memory and never
 *    synchronises, except moe_get_status.  Work is enqueued on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - Weight stacks are stored "out x in" (K-major), one slab per expert:
 *    w_router [E][d]; w1, w_gate, w_up [E+ns][h][d]; w2, w_down [E+ns][d][h],
 *    where ns = num_shared (0 or 1) and the shared expert is slab E.
 *  - Argument errors return before anything is enqueued.  Problems that only
 *    the data reveals (non-finite logits, expert ids out of range, a bounded
 *    device wait that gave up) set bits in the status block inside the
 *    workspace and never trap; read them with moe_get_status.
 *  - ws / ws_bytes: caller-allocated device scratch of at least
 *    moe_workspace_size() bytes, 256-byte aligned.  Its first 256 bytes hold
 *    the status block; moe_workspace_init zeroes it.  Calls that share one
 *    workspace must be ordered on one stream.
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
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size or inconsistent desc */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented combination */
  MOE_ERR_WORKSPACE = 3,    /* ws NULL, misaligned or smaller than needed */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_STATUS = 5 /* moe_get_status found error bits set */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2 } moe_dtype;
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score;
typedef enum { MOE_ACT_GELU = 0, MOE_ACT_SWIGLU = 1 } moe_act;

/* status block bits (moe_get_status flags) */
#define MOE_STATUS_NONFINITE_LOGIT 0x1u /* a router logit was NaN or +-inf */
#define MOE_STATUS_BAD_EXPERT_ID 0x2u   /* moe_permute saw an id outside [0,E) */
#define MOE_STATUS_TIMEOUT 0x4u         /* a bounded device wait gave up */
#define MOE_STATUS_BAD_GROUP 0x8u       /* a group table entry out of range */
#define MOE_STATUS_DEBUG_CHECK 0x10u    /* an internal invariant check failed (the MOE_DEBUG
                                           build's checks; the re-route assignment's epoch bound) */

/* counters (moe_get_status counters[], MOE_NUM_COUNTERS entries) */
#define MOE_CNT_NONFINITE 0   /* tokens with a non-finite logit */
#define MOE_CNT_BAD_ID 1      /* slots with an out-of-range expert id */
#define MOE_CNT_TIMEOUT 2     /* CTAs that gave up a wait */
#define MOE_CNT_OVERFLOW_ROWS 3 /* rows routed to the overflow region */
#define MOE_CNT_REROUTED 4    /* slots moved by over-capacity re-routing */
#define MOE_NUM_COUNTERS 8

/*
 * Layer shape and options.
 *   num_tokens S, d_model d, num_experts E (routed), top_k K, d_ff h.
 *   score_fn: MOE_SCORE_SOFTMAX -- selection key = logit (+ sel_bias);
 *               gates = softmax over the K selected logits (renormalize=1,
 *               the TopK(-inf)-then-Softmax form of 11.1.1) or the full
 *               softmax probability (renormalize=0);
 *             MOE_SCORE_SIGMOID -- s = sigmoid(logit), key = s + sel_bias
 *               (ybb.press "MoE 推理工程深层实战" 2.3, aux-loss-free bias,
 *               used for selection only); gates = s_k / sum_j s_j
 *               (renormalize=1) or s_k.
 *   num_groups, topk_groups: group-limited selection (2.3 of the same page:
 *     group score = sum of the group's keys, keep the topk_groups best
 *     groups, select the K experts inside them).  1,1 = no group limit.
 *     E/num_groups must be a power of two.
 *   num_shared: 0, or 1 always-on shared expert with gate 1 (slab E).
 *   activation: MOE_ACT_GELU  E(x) = GeLU_erf(x W1 + b1) W2 + b2 (11.1.2);
 *               MOE_ACT_SWIGLU E(x) = (SiLU(x Wg) * (x Wu)) Wd.
 *   act_dtype: dtype of x, w_router, y and the intermediates (F32 or BF16).
 *   weight_dtype: dtype of the expert weights (F32, BF16 or E4M3; E4M3
 *     needs the per-output-channel scales s_gate, s_up, s_down).
 *   capacity: 0 = unbounded; C > 0 = at most C rows per expert in the
 *     primary block, the rest in an overflow region (ybb.press 2.2,
 *     overflow buffering) whose rows the expert GEMMs process right after
 *     that expert's primary rows.  No token is dropped.
 *   act_quant: 0 = the expert GEMMs compute on the bf16 activations.  With
 *     E4M3 weights (d and h multiples of 16) each bf16 A row is written as two
 *     E4M3 terms with a power-of-two row scale (moe_split_rows_e4m3), exact
 *     but for elements below about 2^-10.8 of the row's largest magnitude,
 *     and the GEMMs multiply the stored weight codes by both terms in one
 *     fp32 sum; otherwise the weights are decoded to bf16 first.
 *     1 = W8A8: each A row of both expert GEMMs
 *     (the permuted tokens, then the bf16 hidden rows) is quantised to E4M3
 *     with one fp32 scale per row (moe_quantize_rows_e4m3) and the GEMMs run
 *     on 8-bit operands, the epilogue applying row and channel scales.  The
 *     pages list E4M3 only as a storage format (ybb.press 3.3); per-row
 *     activation scaling is this library's reading.  Needs BF16 act, E4M3
 *     weights, SWIGLU, d and h multiples of 16.
 *   reroute: 0 = none; 1 = over-capacity re-routing (needs capacity > 0;
 *     jsqmd.com 11.3.3, expert-dropping paragraph: an overloaded expert's excess tokens go
 *     to their next-best expert).  Each expert keeps its first C slots in
 *     (token, k) order; the excess slots, in (token, k) order, move to the
 *     candidate expert (within the token's kept groups) with the highest
 *     selection key that still has room and that the token does not hold
 *     (ties to the lower index); a slot with no such expert keeps its expert
 *     and its overflow row.  Gates are then recomputed over the final
 *     experts.  See moe_reroute.
 *   temperature: softmax temperature tau of soft routing (jsqmd.com 11.3.3,
 *     soft-routing equation y = sum_i softmax(s/tau)_i E_i(x)).  0 means
 *     tau = 1.  With score_fn = MOE_SCORE_SOFTMAX every logit l (router bias
 *     included) becomes z = l / tau, one float32 division; z is the gate
 *     source and, plus sel_bias, the selection key.  A finite tau > 0;
 *     tau != 1 with MOE_SCORE_SIGMOID is MOE_ERR_UNSUPPORTED (the page gives
 *     the temperature for the softmax router only).  K = E, renormalize = 1
 *     and tau give the page's soft routing.
 * Supported: (F32 act, F32 weights, GELU) with E <= 32 on the SIMT path;
 * (BF16 act, BF16 or E4M3 weights, SWIGLU or GELU; E4M3 with SWIGLU only)
 * on the tensor-core path.  E <= 256, K <= min(E, 32), d and h multiples
 * of 8.
 */
typedef struct {
  int32_t num_tokens;
  int32_t d_model;
  int32_t num_experts;
  int32_t top_k;
  int32_t d_ff;
  int32_t score_fn;
  int32_t renormalize;
  int32_t num_groups;
  int32_t topk_groups;
  int32_t num_shared;
  int32_t activation;
  int32_t act_dtype;
  int32_t weight_dtype;
  int32_t capacity;
  int32_t act_quant;
  int32_t reroute;
  float temperature;
} moe_desc;

/* Weights, all DEVICE pointers (see layouts above).  Unused ones may be
 * NULL: router_bias (added to the logits, so it also moves the gates),
 * sel_bias (added to the selection keys only), b1/b2 (GELU only),
 * s_gate/s_up/s_down (E4M3 only, fp32 [E+ns][h], [E+ns][h], [E+ns][d]). */
typedef struct {
  const void *w_router;
  const float *router_bias;
  const float *sel_bias;
  const void *w1;
  const float *b1;
  const void *w2;
  const float *b2;
  const void *w_gate;
  const void *w_up;
  const void *w_down;
  const float *s_gate;
  const float *s_up;
  const float *s_down;
} moe_weights;

/* Number of rows of the routed row space: S*K, or E*C + S*K with capacity
 * (primary block of E*C rows, then the overflow region).  The shared expert,
 * when present, adds S rows after them in the hidden and expert-output
 * buffers.  Host only. */
int64_t moe_routed_rows(const moe_desc *desc);

/* Workspace bytes needed by moe_layer_forward for this desc (the standalone
 * calls need no more).  Host only, no CUDA call. */
moe_status moe_workspace_size(const moe_desc *desc, size_t *bytes);

/* Zero the status block at the start of `ws` (stream-ordered). */
moe_status moe_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Router logits + scoring + top-k (11.1.1; ybb.press 2.3; plumephp.com
 * "MoE 混合专家推理", routing worked example).
 *   x [S][d] act_dtype; logits_in: optional fp32 [S][E] logits used instead
 *   of computing x W_r^T (router_bias is still added to them); x may then be
 *   NULL.  Outputs topk_idx int32 [S][K] (descending key, ties to the lower
 *   expert index; a non-finite key ranks lowest), topk_w fp32 [S][K].
 */
moe_status moe_route(const moe_desc *desc, const moe_weights *w, const void *x, const float *logits_in,
                     int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream);

/*
 * Histogram, prefix scan and stable permutation (11.2.1, data-regrouping paragraph).
 *   topk_idx int32 [S][K] -> counts int32 [E];
 *   offsets int32 [E+1] (exclusive prefix of counts), with capacity
 *     [2(E+1)]: the first E+1 as before, then the exclusive prefix of the
 *     overflow counts max(counts - C, 0);
 *   row_of_slot int32 [S*K]: row of slot t*K+k; rows of one expert follow
 *     slot order (stable); with capacity rows are e*C+r for r < C and
 *     E*C + ovf_offset[e] + (r-C) otherwise;
 *   token_of_row int32 [R] (R = moe_routed_rows), -1 for unused rows;
 *   x_perm [R][d] act_dtype: x_perm[row_of_slot[t*K+k]] = x[t] (rows with
 *     token_of_row = -1 are left untouched).  x and x_perm may be NULL to
 *     compute only the maps.
 */
moe_status moe_permute(const moe_desc *desc, const void *x, const int32_t *topk_idx, int32_t *counts,
                       int32_t *offsets, int32_t *row_of_slot, int32_t *token_of_row, void *x_perm, void *ws,
                       size_t ws_bytes, void *stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory: a runtime whose device-memory budget is fixed at start-up, code
 * running inside an allocator or other callback where a nested
 * cudaMalloc/cudaFree is not allowed, or a loop that must not risk the
 * device-wide synchronisation cudaFree can cause.  The pages have no
 * counterpart of this call; it exists for those callers only.
 *   Same arguments, outputs and results as moe_permute, minus ws/ws_bytes.
 *   The only scratch (per-chunk expert histograms) lives in a 256 KB device
 *   array inside the library, held by every GPU that loads it until exit.
 *   Sizes whose histograms exceed it -- more than 65536 (chunk, expert)
 *   entries, i.e. ceil(S / floor(1024/K)) * E > 65536 -- return
 *   MOE_ERR_WORKSPACE before anything is enqueued.  The first call on a device looks up the
 *   array's device address (make it before any stream capture).  All calls
 *   share the array: calls that overlap on the GPU race.  There is no status
 *   block: an expert id outside [0, E) gets row -1 in row_of_slot.
 *   Allocates nothing and calls no allocating routine.
 */
moe_status moe_permute_static(const moe_desc *desc, const void *x, const int32_t *topk_idx, int32_t *counts,
                              int32_t *offsets, int32_t *row_of_slot, int32_t *token_of_row, void *x_perm,
                              void *stream);

/*
 * Grouped expert FFN (11.1.2: the S*K expert forwards grouped by expert).
 *   x_perm [R][d] rows grouped as offsets describes (layout of moe_permute);
 *   x [S][d]: A operand of the shared expert (NULL when num_shared = 0);
 *   y_perm [R + ns*S][d] act_dtype: row r = E_{expert(r)}(x_perm[r]); rows
 *     R .. R+S-1 hold the shared expert's output for token 0 .. S-1.
 *   The hidden activations live in the workspace.  Rows outside any group
 *   (unused capacity rows) are not written.  With a capacity, each expert's
 *   overflow rows are processed in the same GEMM launches, right after its
 *   primary rows.  With E4M3 weights the A rows of both GEMMs (x_perm rows
 *   and, for the shared expert, x rows; then the hidden rows) are coded per
 *   row into the workspace -- two-term codes (moe_split_rows_e4m3) with
 *   act_quant = 0, W8A8 codes (moe_quantize_rows_e4m3) with act_quant = 1 --
 *   and the GEMMs multiply them with the stored weight codes; the row and
 *   channel scales multiply the fp32 accumulators.  E4M3 weights with d or h
 *   not a multiple of 16 (act_quant = 0) are instead decoded exactly to bf16
 *   into the workspace on every call.
 */
moe_status moe_grouped_ffn(const moe_desc *desc, const moe_weights *w, const void *x_perm,
                           const int32_t *offsets, const void *x, void *y_perm, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * Over-capacity re-routing (desc->reroute = 1, capacity > 0), the step
 * between a capacity-bounded moe_permute and a second moe_permute:
 *   moe_route (writes the selection keys and gate sources of every expert
 *   into ws) -> moe_permute (x may be NULL) -> moe_reroute -> moe_permute
 *   -> moe_grouped_ffn -> moe_combine.
 * moe_layer_forward runs this sequence by itself when desc->reroute = 1.
 *   topk_idx [S][K] int32 (in/out): the slots listed as excess by
 *     row_of_slot (rows >= E*C) are moved as described at moe_desc.reroute;
 *   topk_w [S][K] fp32 (in/out): the gates of every token with a moved slot
 *     are recomputed over its final experts;
 *   counts [E], row_of_slot [S*K]: moe_permute's outputs for this topk_idx.
 * ws must hold the keys written by the last moe_route on it with the same
 * desc.  One CTA runs the assignment (its visit order is serial; it commits
 * chunks of up to 1024 slots at a time).  Moved slots are counted in
 * MOE_CNT_REROUTED.  Errors: MOE_ERR_INVALID_ARG when reroute != 1 or a
 * pointer is NULL, workspace errors as elsewhere.
 */
moe_status moe_reroute(const moe_desc *desc, int32_t *topk_idx, float *topk_w, const int32_t *counts,
                       const int32_t *row_of_slot, void *ws, size_t ws_bytes, void *stream);

/*
 * Per-row E4M3 quantisation of bf16 rows, the activation step of the W8A8
 * path (act_quant = 1), exposed on its own.  For each row i of x [rows][d]
 * (bf16, row-major, DEVICE, 16-byte aligned, d a multiple of 16):
 *   s[i]    = max_j |x[i][j]| / 448 as one fp32 division; 1 when the row is
 *             all zero or holds a NaN;
 *   q[i][j] = E4M3(x[i][j] / s[i]): fp32 division, round to nearest even,
 *             saturating at +-448; NaN -> 0x7F.
 * q [rows][d] uint8 and s [rows] fp32 are caller-owned DEVICE buffers (q
 * 16-byte aligned).  Launches one kernel on `stream`, allocates nothing.
 * rows = 0 is a no-op.  Errors: MOE_ERR_INVALID_ARG for a NULL or misaligned
 * pointer, rows < 0 or d not a positive multiple of 16; MOE_ERR_CUDA when
 * the launch fails.  There is no workspace or status block.
 */
moe_status moe_quantize_rows_e4m3(const void *x, int64_t rows, int32_t d, uint8_t *q, float *s, void *stream);

/*
 * Two-term E4M3 codes of bf16 rows, the activation step of the E4M3-weight
 * path with bf16 activations (act_quant = 0), exposed on its own.  The
 * tensor cores have no bf16 x E4M3 product (ybb.press "MoE 推理工程深层实战"
 * 3.3 gives E4M3 as the expert weights' storage format), so each bf16 value
 * becomes two E4M3 terms that the GEMM multiplies with the weight codes.
 * For each row i of x [rows][d] (bf16, row-major, DEVICE, 16-byte aligned,
 * d a multiple of 16):
 *   k       = the largest integer with max_j |x[i][j]| * 2^k <= 448,
 *             clamped to [-126, 126] (0 for an all-zero row);
 *   v_j     = x[i][j] * 2^k (exact);
 *   q[i][j]     = E4M3(v_j), round to nearest even;
 *   q[i][d + j] = E4M3(v_j - q[i][j]) (the difference exact in fp32);
 *   s[i]    = 2^-k, or NaN when the row holds an infinity or a NaN
 *             (its codes are then all zero).
 * Then q[i][j] + q[i][d+j] = v_j exactly whenever |v_j| >= 1/4; below that
 * the error is at most 2^-10 in v_j.  q [rows][2d] uint8 and s [rows] fp32
 * are caller-owned DEVICE buffers (q 16-byte aligned).  Launches one kernel
 * on `stream`, allocates nothing.  rows = 0 is a no-op.  Errors:
 * MOE_ERR_INVALID_ARG for a NULL or misaligned pointer, rows < 0 or d not a
 * positive multiple of 16; MOE_ERR_CUDA when the launch fails.
 */
moe_status moe_split_rows_e4m3(const void *x, int64_t rows, int32_t d, uint8_t *q, float *s, void *stream);

/*
 * Gate-weighted combine back into token order (11.3.1 step 6; plumephp.com
 * "MoE 混合专家推理", worked-example block: the gate-weighted sum).
 *   y[t] = sum_{k=0..K-1} topk_w[t][k] * y_perm[row_of_slot[t*K+k]]
 *          (+ y_perm[R + t] when num_shared = 1), fp32 sums in k order.
 *   y [S][d] act_dtype.
 */
moe_status moe_combine(const moe_desc *desc, const void *y_perm, const int32_t *row_of_slot,
                       const float *topk_w, void *y, void *ws, size_t ws_bytes, void *stream);

/*
 * The whole layer: route -> permute -> grouped FFN -> combine, enqueued
 * without any host synchronisation.  y [S][d] act_dtype.  topk_idx, topk_w
 * and counts are optional outputs (NULL = keep them in the workspace).
 */
moe_status moe_layer_forward(const moe_desc *desc, const moe_weights *w, const void *x, void *y,
                             int32_t *topk_idx, float *topk_w, int32_t *counts, void *ws, size_t ws_bytes,
                             void *stream);

/*
 * moe_layer_forward that also records caller-created CUDA events on `stream`
 * between its stages, so a caller can time each stage of the real layer call
 * (the same launches as moe_layer_forward, plus the event records).
 * events: MOE_NUM_STAGE_EVENTS cudaEvent_t handles passed as void*, each one
 * NULL (skipped) or an event created on the current device:
 *   [0] before routing             [1] after routing (and re-routing)
 *   [2] after the permutation       [3] before the up-projection GEMM (after
 *   any E4M3 weight decode or coding of the A rows in the FFN)
 *   [4] after the up-projection GEMM   [5] before the down-projection GEMM
 *   [6] after the down-projection GEMM [7] after the combine.
 * Errors as moe_layer_forward; MOE_ERR_CUDA when an event record fails.
 */
#define MOE_NUM_STAGE_EVENTS 8
moe_status moe_layer_forward_timed(const moe_desc *desc, const moe_weights *w, const void *x, void *y,
                                   int32_t *topk_idx, float *topk_w, int32_t *counts, void *ws, size_t ws_bytes,
                                   void *stream, void *const *events);

/*
 * Sliding-window expert load and the aux-loss-free selection-bias update
 * (ybb.press "MoE 推理工程深层实战" 2.3: the bias added to the selection keys
 * is recomputed from a token counter over a sliding window of 1000 tokens,
 * so routing is steered without gradients).  The page
 * prints no update rule; this call applies, per expert, in float32,
 *     sel_bias[e] += gamma * sign(mean - count_e),
 * count_e = (token, k) slots routed to e among the last `window_tokens`
 * tokens, mean = tokens_in_window * K / E.
 *   state: caller-owned device memory of moe_bias_state_size() bytes, zeroed
 *     by moe_bias_state_init before the first update (it holds the window's
 *     expert ids and counts).  The window fills from empty; a batch of S
 *     tokens replaces the S oldest ones (only its last window_tokens tokens
 *     count when S >= window_tokens).  Ids outside [0, E) are not counted.
 *   topk_idx int32 [S][K] (e.g. moe_route's output); sel_bias fp32 [E] is
 *   updated in place; window_counts int32 [E] (optional) receives count_e.
 *   One window per state; calls on one state must be stream-ordered.
 */
moe_status moe_bias_state_size(const moe_desc *desc, int32_t window_tokens, size_t *bytes);
moe_status moe_bias_state_init(void *state, size_t state_bytes, void *stream);
moe_status moe_update_sel_bias(const moe_desc *desc, const int32_t *topk_idx, int32_t window_tokens, float gamma,
                               void *state, size_t state_bytes, float *sel_bias, int32_t *window_counts,
                               void *stream);

/*
 * Load report of one routing, computed on the device from the per-expert
 * counts (moe_permute's or moe_layer_forward's counts output).  It gathers
 * what the pages ask to watch: the max/mean expert load (jsqmd.com 11.2.3,
 * 1 when balanced, 3-5 in practice), the standard deviation of the expert
 * loads and the token drop rate (ybb.press "MoE 推理工程深层实战" 1.2, table
 * of inference metrics), the rows above the capacity (ybb.press 2.2) and the
 * routing histogram itself (plumephp.com "MoE 混合专家推理", verification
 * block).
 *   counts int32 [E] DEVICE; stats double [MOE_NUM_LOAD_STATS] DEVICE,
 *   caller-owned, written as
 *     [MOE_LS_MAX_OVER_MEAN] max_e counts[e] / mean   (0 when S*K = 0)
 *     [MOE_LS_STD]           sqrt(sum_e (counts[e] - mean)^2 / E)
 *     [MOE_LS_MEAN]          mean = S*K / E
 *     [MOE_LS_MAX]           max_e counts[e]
 *     [MOE_LS_OVERFLOW_ROWS] sum_e max(counts[e] - capacity, 0) (0 without
 *                            a capacity): rows in the overflow region
 *     [MOE_LS_DROPPED]       S*K - sum_e counts[e]: slots that got no row.
 *                            The layer drops no token, so this is 0 unless
 *                            an expert id was outside [0, E).
 * One kernel on `stream`; no workspace.  Errors: MOE_ERR_INVALID_ARG for an
 * invalid desc or a NULL / misaligned pointer, MOE_ERR_CUDA for a failed
 * launch.
 */
#define MOE_LS_MAX_OVER_MEAN 0
#define MOE_LS_STD 1
#define MOE_LS_MEAN 2
#define MOE_LS_MAX 3
#define MOE_LS_OVERFLOW_ROWS 4
#define MOE_LS_DROPPED 5
#define MOE_NUM_LOAD_STATS 6
moe_status moe_load_stats(const moe_desc *desc, const int32_t *counts, double *stats, void *stream);

/* Synchronise `stream`, copy the status block to the host.  flags: OR of
 * MOE_STATUS_* bits; counters: MOE_NUM_COUNTERS int32 (may be NULL).
 * Returns MOE_ERR_DEVICE_STATUS when any error bit is set. */
moe_status moe_get_status(const void *ws, void *stream, uint32_t *flags, int32_t *counters);

/* Static description of a status code. */
const char *moe_strerror(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
