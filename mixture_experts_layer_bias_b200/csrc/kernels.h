// Host-side launchers of the MoE layer kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

struct StatusBlock;

// --- routing ---------------------------------------------------------------
// Router logits: E <= 32 are computed inside the routing kernels (a CTA per
// token for S <= 512; else, with W_r of at most kRouteWSmemBytes, tensor-core
// products over 16 tokens per CTA with W_r read from L1/L2 (bf16), or warps
// streaming token rows against a copy of W_r in shared memory (fp32));
// otherwise (E > 32, or a larger W_r when S > 512, which every CTA would read
// again) one logits GEMM into the workspace first, then the selection.
constexpr int kRouteWSmemBytes = 64 << 10;
inline bool route_logits_first(int64_t S, int64_t E, int64_t d, int elem_bytes) {
  return E > 32 || (S > 512 && E * d * elem_bytes > kRouteWSmemBytes);
}

struct RouteArgs {
  int S, d, E, K;
  int score_fn, renormalize, num_groups, topk_groups;
  float tau;                // softmax temperature: logits are divided by it (1 = none)
  int act_dtype;
  const void* x;            // [S][d] (unused when logits given)
  const void* w_router;     // [E][d]
  const float* logits;      // [S][E] fp32 or nullptr (then computed)
  float* logits_scratch;    // [S][E] fp32 scratch (route_logits_first)
  const float* router_bias; // [E] or nullptr
  const float* sel_bias;    // [E] or nullptr
  int32_t* topk_idx;        // [S][K]
  float* topk_w;            // [S][K]
  StatusBlock* status;
  int num_sms;
  float* cand_key_out;      // optional [S][E]: candidate keys (-inf for non-candidates), for re-routing
  float* score_out;         // optional [S][E]: gate sources (logits or sigmoid scores), with cand_key_out
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream);

// --- over-capacity re-routing ------------------------------------------------
// Excess slots (row_of_slot >= E*C after a capacity-bounded permutation) move,
// in (token, k) order, to the best-keyed candidate expert with room that the
// token does not hold; changed[t] marks tokens with a moved slot.  A multi-CTA
// pick kernel, one CTA running the epochs, a multi-CTA apply kernel.
struct RerouteScratch {
  int32_t* pick;      // [S*K], 16-byte aligned
  int8_t* pick8;      // [S*K] rounded up to 16, 16-byte aligned: a byte copy of the picks (E <= 127)
  int32_t* ex;        // [S*K], 16-byte aligned: the excess slots
  int32_t* ex_count;  // one int
  int32_t* claim;     // [S]
  int32_t* list;      // [S]
};
cudaError_t launch_reroute_assign(int S, int E, int K, int capacity, int32_t* topk_idx, const float* cand_key,
                                  const int32_t* counts, const int32_t* row_of_slot, const RerouteScratch& w,
                                  int32_t* changed, StatusBlock* status, cudaStream_t stream);
// Gates of the tokens marked in changed[], recomputed over their final experts
// from the gate sources (the same formulas as the routing kernels).
cudaError_t launch_reroute_gates(int S, int E, int K, int score_fn, int renormalize, const float* score,
                                 const int32_t* changed, const int32_t* topk_idx, float* topk_w, cudaStream_t stream);

// --- grouping by expert -----------------------------------------------------
// Group table entry of the grouped GEMMs: rows [a_row0, a_row0 + rows) of the
// A operand, written to rows [out_row0, out_row0 + rows) of the output, all
// with the weights of slab `expert`.
struct GroupEntry {
  int32_t a_row0, out_row0, rows, expert;
};

struct PermuteArgs {
  int S, d, E, K, capacity, act_dtype;
  const int32_t* topk_idx;   // [S][K]
  int32_t* chunk_hist;       // [num_chunks][E] scratch
  int32_t* counts;           // [E]
  int32_t* offsets;          // [E+1] (+ [E+1] overflow offsets with capacity)
  int32_t* row_of_slot;      // [S*K]
  int32_t* token_of_row;     // [R]
  const void* x;             // [S][d] or nullptr
  void* x_perm;              // [R][d] or nullptr
  int64_t num_rows;          // R
  StatusBlock* status;
  // optional: also write the GEMM group table (see GroupEntry)
  GroupEntry* g1;
  int num_shared;
};
int permute_num_chunks(int S, int K);
int permute_tokens_per_chunk(int K);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t stream);

// Build the group table from offsets: E routed groups, or with a capacity
// 2E (expert e's primary group at 2e, its overflow group at 2e + 1), then
// the shared expert; E + ns or 2E + ns entries.
cudaError_t launch_build_groups(int S, int E, int K, int capacity, int num_shared, const int32_t* offsets,
                                GroupEntry* g1, StatusBlock* status, cudaStream_t stream);

// --- grouped expert GEMMs ----------------------------------------------------
enum Epilogue { EPI_SWIGLU = 0, EPI_GELU_BIAS = 1, EPI_BIAS = 2, EPI_NONE = 3 };

struct GemmArgs {
  int epilogue;
  const GroupEntry* groups;  // nullptr: a single group of max_total_rows rows (slab 0, rows from 0)
  int num_groups;
  int shared_slab;          // slab index whose A rows come from a_shared, -1 = none
  int a_rows_from_out;      // 1: A row = out_row0 + r (down projection), 0: a_row0 + r
  const void* a;            // A operand [a_rows][K]
  int64_t a_rows;
  const void* a_shared;     // shared-expert A operand [a_shared_rows][K] (up projection)
  int64_t a_shared_rows;
  const void* b0;           // weights [slabs * n_per_slab][K] (gate for SwiGLU)
  const void* b1;           // up weights (SwiGLU), else unused
  int64_t b_rows;           // slabs * n_per_slab
  int n_per_slab;           // N rows of one slab (h or d)
  int N, K;                 // output columns, reduction length
  const float* bias;        // [slabs][N] or nullptr
  const float* scale0;      // per-output-channel scale [slabs][N] (gate / plain)
  const float* scale1;      // per-output-channel scale [slabs][N] (up)
  void* out;                // [out_rows][N]
  int64_t out_rows;
  int out_f32;              // 1: fp32 output, 0: bf16
  int64_t max_total_rows;   // upper bound of the rows of all groups together
  int64_t max_group_rows;   // upper bound of the rows of one group
  float* partial;           // split-K partial sums (nullptr = no split-K)
  int64_t partial_bytes;    // size of `partial`
  int* ksplit_out;          // device int: the split the GEMM chose (read by the finalize kernel)
  int fp8;                  // 1: A and B are E4M3 (kind::f8f6f4); A rows scaled by row_scale
  int a_terms;              // fp8: 2 = A rows hold two-term codes [c1 | c2] (2K codes), summed in one accumulator
  const float* row_scale;        // [a rows] per-row scale of A (fp8 only)
  const float* row_scale_shared; // [S] per-row scale of the shared expert's A rows (fp8 only)
  StatusBlock* status;
};
cudaError_t launch_grouped_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t stream);
namespace gemm {
struct TcParams;
}
cudaError_t launch_grouped_gemm_single(const GemmArgs& a, const gemm::TcParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_grouped_gemm_f32(const GemmArgs& a, cudaStream_t stream);

// FP8-E4M3 weight slabs -> bf16 (exact)
cudaError_t launch_dequant_e4m3(const uint8_t* q, void* out_bf16, int64_t n, cudaStream_t stream);

// --- E4M3 activations (W8A8) -------------------------------------------------
// Per-row quantisation of bf16 rows.  terms = 1 (W8A8): s = amax / 448 (1
// for an all-zero row or a row holding a NaN), q = RNE satfinite E4M3
// (x / s), both float32 divisions; rows of d codes.  terms = 2 (E4M3
// weights, bf16 activations): two-term codes c1 | c2 with x * 2^k = c1 + c2
// and s = 2^-k (quant.cu); rows of 2d codes.
cudaError_t launch_quantize_rows(const void* src, uint8_t* dst, float* scale, int64_t rows, int d, int terms,
                                 cudaStream_t stream);
// The row gather of the permutation fused with that quantisation: token t's
// codes and scale go to rows row_of_slot[t*K + k] (>= 0) of q_perm / s_perm
// and, when q_x is given, to row t of q_x / s_x.
cudaError_t launch_gather_quantize(int S, int d, int K, const int32_t* row_of_slot, const void* x, uint8_t* q_perm,
                                   float* s_perm, uint8_t* q_x, float* s_x, int terms, cudaStream_t stream);
// The same for the rows of a group table: rows a_row0 + r (or out_row0 + r
// with use_out_rows) of src, at most dst_rows; the shared-expert group's
// rows come from src_shared and go to dst_shared / scale_shared (index r,
// at most shared_rows).  max_total_rows bounds the rows of all groups
// together (it sizes the grid).
cudaError_t launch_quantize_group_rows(const GroupEntry* groups, int num_groups, int use_out_rows, int shared_slab,
                                       const void* src, uint8_t* dst, float* scale, int64_t dst_rows,
                                       const void* src_shared, uint8_t* dst_shared, float* scale_shared,
                                       int64_t shared_rows, int d, int64_t max_total_rows, int terms,
                                       StatusBlock* status, cudaStream_t stream);

// --- sliding-window load and selection-bias update ---------------------------
size_t bias_state_bytes(int E, int K, int window);
cudaError_t launch_bias_update(int S, int E, int K, int window, const int32_t* topk_idx, float gamma, void* state,
                               float* sel_bias, int32_t* window_counts, cudaStream_t stream);

// --- load report -------------------------------------------------------------
// MOE_NUM_LOAD_STATS doubles from counts[E] (one CTA; see moe_load_stats).
cudaError_t launch_load_stats(int E, int64_t slots, int capacity, const int32_t* counts, double* out,
                              cudaStream_t stream);

// --- combine -----------------------------------------------------------------
struct CombineArgs {
  int S, d, K, act_dtype;
  const void* y_perm;
  const int32_t* row_of_slot;
  const float* topk_w;
  int64_t shared_row0;  // -1 = no shared expert
  void* y;
  int64_t num_rows;     // rows of y_perm (debug builds check row_of_slot against it)
  StatusBlock* status;  // debug builds report a row outside y_perm here (may be nullptr)
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

// --- MOE_DEBUG builds ----------------------------------------------------------
// Invariants of a permutation: offsets[e+1] - offsets[e] = counts[e] (and the
// overflow split with a capacity), every row_of_slot in [-1, R), token_of_row
// the inverse map.  A violation sets MOE_STATUS_DEBUG_CHECK.  Launched after
// every permutation of a debug build only.
cudaError_t launch_debug_check_permutation(int S, int E, int K, int capacity, const int32_t* counts,
                                           const int32_t* offsets, const int32_t* row_of_slot,
                                           const int32_t* token_of_row, int64_t num_rows, StatusBlock* status,
                                           cudaStream_t stream);

}  // namespace moe
