// C ABI of the MoE layer forward: argument checks, workspace layout and the
// launch sequence (declarations and contracts in include/moe.h).
//
// The layer follows jsqmd.com "第11章 MoE模型推理" 11.1.1-11.1.2 and 11.2.1:
// route (router + TopK), regroup the S*K token slots by expert, run each
// expert's FFN over its rows as one grouped GEMM, restore token order with
// the gate-weighted sum.  Nothing here allocates or synchronises (except
// moe_get_status); every launch goes to the caller's stream.
#include <nvtx3/nvToolsExt.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

// NVTX range around each entry point and each stage of the layer call (host
// timeline; a profiler can filter the kernels launched inside a range).  The
// calls cost a few nanoseconds when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

struct Layout {
  size_t status, logits, chunk_hist, groups, counts, offsets, topk_idx, topk_w, row_of_slot,
      token_of_row, x_perm, hidden, y_perm, wdeq, ksplit, partial, partial_bytes, qa, sa, qas, sas, qh, sh, rr_key,
      rr_score, rr_ex, rr_pick8, rr_exl, rr_excount, rr_claim, rr_list, rr_changed, total;
};

// Split-K of the tensor-core GEMMs is available to small row spaces (decode-
// sized batches), where too few output tiles exist to occupy every SM.  The
// partial sums take at most this much workspace.
constexpr int64_t kSplitRowsMax = 4096;
constexpr int64_t kPartialBudget = int64_t(256) << 20;

int64_t routed_rows(const moe_desc& d) {
  const int64_t sk = static_cast<int64_t>(d.num_tokens) * d.top_k;
  return d.capacity > 0 ? static_cast<int64_t>(d.num_experts) * d.capacity + sk : sk;
}

size_t act_bytes(const moe_desc& d) { return d.act_dtype == MOE_F32 ? 4 : 2; }

// Codes of the expert GEMMs' A rows: 0 = the GEMMs read bf16 (or fp32) rows;
// 1 = W8A8 (one E4M3 code per element, scale amax / 448); 2 = E4M3 weights
// with bf16 activations: each bf16 element as two E4M3 terms with a
// power-of-two row scale (quant.cu), so the GEMMs multiply the stored weight
// codes directly.  Rows must be whole 16-byte pieces of codes (d and h
// multiples of 16); otherwise the weights are decoded to bf16 first.
int a_terms(const moe_desc& d) {
  if (d.act_quant == 1) return 1;
  if (d.weight_dtype == MOE_E4M3 && d.act_dtype == MOE_BF16 && d.d_model % 16 == 0 && d.d_ff % 16 == 0) return 2;
  return 0;
}

Layout make_layout(const moe_desc& d) {
  Layout L;
  const int64_t S = d.num_tokens, E = d.num_experts, K = d.top_k, h = d.d_ff, dm = d.d_model;
  const int64_t R = routed_rows(d);
  const int64_t Rt = R + static_cast<int64_t>(d.num_shared) * S;
  const int64_t nch = permute_num_chunks(static_cast<int>(S), static_cast<int>(K));
  const size_t ab = act_bytes(d);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.status = take(kAlign);
  L.logits = take(route_logits_first(S, E, dm, static_cast<int>(act_bytes(d))) ? static_cast<size_t>(S * E) * 4 : 0);
  L.chunk_hist = take(static_cast<size_t>(nch * E) * 4);
  L.groups = take(static_cast<size_t>(2 * E + 1) * sizeof(GroupEntry));
  L.counts = take(static_cast<size_t>(E) * 4);
  L.offsets = take(static_cast<size_t>(2 * (E + 1)) * 4);
  L.topk_idx = take(static_cast<size_t>(S * K) * 4);
  L.topk_w = take(static_cast<size_t>(S * K) * 4);
  L.row_of_slot = take(static_cast<size_t>(S * K) * 4);
  L.token_of_row = take(static_cast<size_t>(R) * 4);
  // (E4M3 A rows: the row gather writes codes, no bf16 copy of the permuted rows)
  L.x_perm = take(a_terms(d) ? 0 : static_cast<size_t>(R * dm) * ab);
  L.hidden = take(static_cast<size_t>(Rt * h) * ab);
  L.y_perm = take(static_cast<size_t>(Rt * dm) * ab);
  const int terms = a_terms(d);
  L.wdeq = take(d.weight_dtype == MOE_E4M3 && terms == 0 ? static_cast<size_t>((E + d.num_shared) * 3 * h * dm) * 2
                                                          : 0);
  // E4M3 A rows (W8A8, or two-term codes): codes and row scales of the up
  // GEMM's A rows (permuted tokens; the shared expert's tokens) and of the
  // down GEMM's (hidden rows)
  L.qa = take(static_cast<size_t>(terms * R * dm));
  L.sa = take(terms ? static_cast<size_t>(R) * 4 : 0);
  L.qas = take(d.num_shared ? static_cast<size_t>(terms * S * dm) : 0);
  L.sas = take(terms && d.num_shared ? static_cast<size_t>(S) * 4 : 0);
  L.qh = take(static_cast<size_t>(terms * Rt * h));
  L.sh = take(terms ? static_cast<size_t>(Rt) * 4 : 0);
  // re-routing: every expert's selection key and gate source, the slots' picks, the excess-slot list and
  // its count, token claims and lists, changed tokens
  const bool rr = d.reroute == 1;
  L.rr_key = take(rr ? static_cast<size_t>(S * E) * 4 : 0);
  L.rr_score = take(rr ? static_cast<size_t>(S * E) * 4 : 0);
  L.rr_ex = take(rr ? static_cast<size_t>(S * K) * 4 : 0);
  L.rr_pick8 = take(rr ? (static_cast<size_t>(S * K) + 15) & ~size_t(15) : 0);
  L.rr_exl = take(rr ? static_cast<size_t>(S * K) * 4 : 0);
  L.rr_excount = take(rr ? 4 : 0);
  L.rr_claim = take(rr ? static_cast<size_t>(S) * 4 : 0);
  L.rr_list = take(rr ? static_cast<size_t>(S) * 4 : 0);
  L.rr_changed = take(rr ? static_cast<size_t>(S) * 4 : 0);
  L.ksplit = take(kAlign);
  L.partial_bytes = 0;
  if (d.act_dtype == MOE_BF16 && Rt > 0 && Rt <= kSplitRowsMax) {
    const int64_t up_cols = d.activation == MOE_ACT_SWIGLU ? 2 * h : h;
    const int64_t per_split = Rt * (up_cols > dm ? up_cols : dm) * 4;
    int64_t bytes = 16 * per_split;
    if (bytes > kPartialBudget) bytes = kPartialBudget;
    if (bytes >= 2 * per_split) L.partial_bytes = static_cast<size_t>(bytes);
  }
  L.partial = take(L.partial_bytes);
  L.total = o;
  return L;
}

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

moe_status validate(const moe_desc* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->num_tokens < 0 || d->d_model <= 0 || d->d_model % 8 != 0 || d->d_ff <= 0 || d->d_ff % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (d->num_experts < 1 || d->num_experts > 256) return MOE_ERR_INVALID_ARG;
  if (d->top_k < 1 || d->top_k > d->num_experts || d->top_k > 32) return MOE_ERR_INVALID_ARG;
  if (d->score_fn != MOE_SCORE_SOFTMAX && d->score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (d->renormalize != 0 && d->renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (d->num_groups < 1 || d->num_experts % d->num_groups != 0) return MOE_ERR_INVALID_ARG;
  if (d->topk_groups < 1 || d->topk_groups > d->num_groups) return MOE_ERR_INVALID_ARG;
  const int gs = d->num_experts / d->num_groups;
  if (d->num_groups > 1 && !is_pow2(gs)) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(d->topk_groups) * gs < d->top_k) return MOE_ERR_INVALID_ARG;
  if (d->num_shared != 0 && d->num_shared != 1) return MOE_ERR_INVALID_ARG;
  if (d->activation != MOE_ACT_GELU && d->activation != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (d->act_dtype != MOE_F32 && d->act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (d->weight_dtype != MOE_F32 && d->weight_dtype != MOE_BF16 && d->weight_dtype != MOE_E4M3)
    return MOE_ERR_INVALID_ARG;
  if (d->capacity < 0) return MOE_ERR_INVALID_ARG;
  if (d->act_quant != 0 && d->act_quant != 1) return MOE_ERR_INVALID_ARG;
  if (d->reroute != 0 && d->reroute != 1) return MOE_ERR_INVALID_ARG;
  if (d->reroute == 1 && d->capacity <= 0) return MOE_ERR_INVALID_ARG;
  // temperature: 0 (= 1) or a finite positive float (the comparison also rejects NaN)
  if (!(d->temperature >= 0.0f) || d->temperature > 3.0e38f) return MOE_ERR_INVALID_ARG;
  // row indices are int32 on the device
  const int64_t rows = routed_rows(*d) + static_cast<int64_t>(d->num_shared) * d->num_tokens;
  if (rows > (int64_t(1) << 31) - 1) return MOE_ERR_INVALID_ARG;
  // implemented combinations
  if (d->act_dtype == MOE_F32) {
    if (d->weight_dtype != MOE_F32 || d->activation != MOE_ACT_GELU) return MOE_ERR_UNSUPPORTED;
  } else {
    if (d->weight_dtype == MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (d->weight_dtype == MOE_E4M3 && d->activation != MOE_ACT_SWIGLU) return MOE_ERR_UNSUPPORTED;
  }
  if (d->score_fn == MOE_SCORE_SIGMOID && d->temperature != 0.0f && d->temperature != 1.0f)
    return MOE_ERR_UNSUPPORTED;
  if (d->act_quant == 1 && (d->act_dtype != MOE_BF16 || d->weight_dtype != MOE_E4M3 ||
                            d->activation != MOE_ACT_SWIGLU || d->d_model % 16 != 0 || d->d_ff % 16 != 0))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ws(const moe_desc& d, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_WORKSPACE;
  if (ws_bytes < make_layout(d).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// SM count of the current device, queried once per device ordinal.
int num_sms() {
  static int cache[64] = {0};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  if (dev < 64) cache[dev] = n;
  return n;
}

RouteArgs route_args(const moe_desc& d, const moe_weights* w, const void* x, const float* logits_in,
                     int32_t* topk_idx, float* topk_w, void* ws) {
  const Layout L = make_layout(d);
  RouteArgs a{};
  a.S = d.num_tokens;
  a.d = d.d_model;
  a.E = d.num_experts;
  a.K = d.top_k;
  a.score_fn = d.score_fn;
  a.renormalize = d.renormalize;
  a.tau = d.temperature == 0.0f ? 1.0f : d.temperature;
  a.num_groups = d.num_groups;
  a.topk_groups = d.topk_groups;
  a.act_dtype = d.act_dtype;
  a.x = x;
  a.w_router = w != nullptr ? w->w_router : nullptr;
  a.logits = logits_in;
  a.logits_scratch = at<float>(ws, L.logits);
  a.router_bias = w != nullptr ? w->router_bias : nullptr;
  a.sel_bias = w != nullptr ? w->sel_bias : nullptr;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.status = at<StatusBlock>(ws, L.status);
  a.num_sms = num_sms();
  if (d.reroute == 1) {
    a.cand_key_out = at<float>(ws, L.rr_key);
    a.score_out = at<float>(ws, L.rr_score);
  }
  return a;
}

moe_status route_impl(const moe_desc& d, const moe_weights* w, const void* x, const float* logits_in,
                      int32_t* topk_idx, float* topk_w, void* ws, cudaStream_t st) {
  return cuda_status(launch_route(route_args(d, w, x, logits_in, topk_idx, topk_w, ws), st));
}

PermuteArgs permute_args(const moe_desc& d, const void* x, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                         int32_t* row_of_slot, int32_t* token_of_row, void* x_perm, void* ws, bool write_groups) {
  const Layout L = make_layout(d);
  PermuteArgs a{};
  a.S = d.num_tokens;
  a.d = d.d_model;
  a.E = d.num_experts;
  a.K = d.top_k;
  a.capacity = d.capacity;
  a.act_dtype = d.act_dtype;
  a.topk_idx = topk_idx;
  a.chunk_hist = at<int32_t>(ws, L.chunk_hist);
  a.counts = counts;
  a.offsets = offsets;
  a.row_of_slot = row_of_slot;
  a.token_of_row = token_of_row;
  a.x = x;
  a.x_perm = x_perm;
  a.num_rows = routed_rows(d);
  a.status = at<StatusBlock>(ws, L.status);
  if (write_groups) {
    a.g1 = at<GroupEntry>(ws, L.groups);
    a.num_shared = d.num_shared;
  }
  return a;
}

// A MOE_DEBUG build checks the permutation's invariants after it (a no-op
// otherwise: nothing is launched).
moe_status debug_check(const PermuteArgs& a, cudaStream_t st) {
  return cuda_status(launch_debug_check_permutation(a.S, a.E, a.K, a.capacity, a.counts, a.offsets, a.row_of_slot,
                                                    a.token_of_row, a.num_rows, a.status, st));
}

moe_status permute_impl(const moe_desc& d, const void* x, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                        int32_t* row_of_slot, int32_t* token_of_row, void* x_perm, void* ws, cudaStream_t st,
                        bool write_groups = false) {
  const PermuteArgs a =
      permute_args(d, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm, ws, write_groups);
  const moe_status s = cuda_status(launch_permute(a, st));
  return s != MOE_OK ? s : debug_check(a, st);
}

// Record stage event `i` of `events` (moe_layer_forward_timed), if given.
bool record(void* const* events, int i, cudaStream_t st) {
  if (events == nullptr || events[i] == nullptr) return true;
  return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
}

moe_status ffn_impl(const moe_desc& d, const moe_weights& w, const void* x_perm, const int32_t* offsets, const void* x,
                    void* y_perm, void* ws, cudaStream_t st, bool groups_ready = false, bool a_quantized = false,
                    void* const* events = nullptr) {
  const Layout L = make_layout(d);
  const int S = d.num_tokens, E = d.num_experts, h = d.d_ff, dm = d.d_model;
  if (S == 0) return MOE_OK;
  const int64_t R = routed_rows(d);
  const int64_t Rt = R + static_cast<int64_t>(d.num_shared) * S;
  StatusBlock* status = at<StatusBlock>(ws, L.status);
  GroupEntry* g1 = at<GroupEntry>(ws, L.groups);
  cudaError_t err = cudaSuccess;
  if (!groups_ready) {
    err = launch_build_groups(S, E, d.top_k, d.capacity, d.num_shared, offsets, g1, status, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  const int slabs = E + d.num_shared;
  void* hidden = at<void>(ws, L.hidden);

  GemmArgs up{};
  up.groups = g1;
  // with a capacity the overflow groups sit right behind each expert's primary group
  up.num_groups = (d.capacity > 0 ? 2 * E : E) + d.num_shared;
  up.shared_slab = d.num_shared ? E : -1;
  up.a_rows_from_out = 0;
  up.a = x_perm;
  up.a_rows = R;
  up.a_shared = d.num_shared ? x : nullptr;
  up.a_shared_rows = d.num_shared ? S : 0;
  up.n_per_slab = h;
  up.b_rows = static_cast<int64_t>(slabs) * h;
  up.N = h;
  up.K = dm;
  up.out = hidden;
  up.out_rows = Rt;
  up.out_f32 = d.act_dtype == MOE_F32;
  up.max_total_rows = static_cast<int64_t>(S) * d.top_k + static_cast<int64_t>(d.num_shared) * S;
  up.max_group_rows = S;
  up.status = status;
  up.partial = L.partial_bytes ? at<float>(ws, L.partial) : nullptr;
  up.partial_bytes = static_cast<int64_t>(L.partial_bytes);
  up.ksplit_out = at<int>(ws, L.ksplit);

  GemmArgs down = up;
  down.a_rows_from_out = 1;
  down.shared_slab = -1;
  down.a = hidden;
  down.a_rows = Rt;
  down.a_shared = nullptr;
  down.a_shared_rows = 0;
  down.n_per_slab = dm;
  down.b_rows = static_cast<int64_t>(slabs) * dm;
  down.N = dm;
  down.K = h;
  down.out = y_perm;

  if (d.act_dtype == MOE_F32) {
    up.epilogue = EPI_GELU_BIAS;
    up.b0 = w.w1;
    up.bias = w.b1;
    down.epilogue = EPI_BIAS;
    down.b0 = w.w2;
    down.bias = w.b2;
  } else {
    const void *wg = w.w_gate, *wu = w.w_up, *wd = w.w_down, *w1 = w.w1, *w2 = w.w2;
    if (a_terms(d) > 0) {
      // E4M3 weights read as they are by kind::f8f6f4 GEMMs; the A rows are
      // E4M3 codes (W8A8: one per element; bf16 activations: two terms per
      // element), made per row right before each GEMM (below) or by the row
      // gather; the epilogue applies the row and the channel scales
      up.fp8 = down.fp8 = 1;
      up.a_terms = down.a_terms = a_terms(d);
      up.scale0 = w.s_gate;
      up.scale1 = w.s_up;
      down.scale0 = w.s_down;
      up.a = at<void>(ws, L.qa);
      up.row_scale = at<float>(ws, L.sa);
      up.a_shared = d.num_shared ? at<void>(ws, L.qas) : nullptr;
      up.row_scale_shared = d.num_shared ? at<float>(ws, L.sas) : nullptr;
      down.a = at<void>(ws, L.qh);
      down.row_scale = at<float>(ws, L.sh);
      down.row_scale_shared = nullptr;
    } else if (d.weight_dtype == MOE_E4M3) {
      // exact E4M3 -> bf16 decode of this call's weights into the workspace
      // (many rows per expert, or d or h not a multiple of 16); the
      // per-channel scales are applied to the fp32 accumulators in the
      // epilogues
      const int64_t n_up = static_cast<int64_t>(slabs) * h * dm;
      char* base = at<char>(ws, L.wdeq);
      void* dg = base;
      void* du = base + n_up * 2;
      void* dd = base + 2 * n_up * 2;
      if ((err = launch_dequant_e4m3(static_cast<const uint8_t*>(wg), dg, n_up, st)) != cudaSuccess ||
          (err = launch_dequant_e4m3(static_cast<const uint8_t*>(wu), du, n_up, st)) != cudaSuccess ||
          (err = launch_dequant_e4m3(static_cast<const uint8_t*>(wd), dd, n_up, st)) != cudaSuccess)
        return MOE_ERR_CUDA;
      wg = dg;
      wu = du;
      wd = dd;
      up.scale0 = w.s_gate;
      up.scale1 = w.s_up;
      down.scale0 = w.s_down;
    }
    if (d.activation == MOE_ACT_SWIGLU) {
      up.epilogue = EPI_SWIGLU;
      up.b0 = wg;
      up.b1 = wu;
      down.epilogue = EPI_NONE;
      down.b0 = wd;
    } else {
      up.epilogue = EPI_GELU_BIAS;
      up.b0 = w1;
      up.bias = w.b1;
      down.epilogue = EPI_BIAS;
      down.b0 = w2;
      down.bias = w.b2;
    }
  }
  const int sms = num_sms();
  auto run = [&](const GemmArgs& g) {
    return d.act_dtype == MOE_F32 ? launch_grouped_gemm_f32(g, st) : launch_grouped_gemm_tc(g, sms, st);
  };
  // E4M3 A rows: codes + row scales of the A rows a GEMM over `g` reads
  const int terms = a_terms(d);
  auto quant_up = [&](const GemmArgs& g) {
    return launch_quantize_group_rows(g.groups, g.num_groups, 0, g.shared_slab, x_perm, at<uint8_t>(ws, L.qa),
                                      at<float>(ws, L.sa), R, x, d.num_shared ? at<uint8_t>(ws, L.qas) : nullptr,
                                      d.num_shared ? at<float>(ws, L.sas) : nullptr, S, dm, g.max_total_rows, terms,
                                      status, st);
  };
  auto quant_down = [&](const GemmArgs& g) {
    return launch_quantize_group_rows(g.groups, g.num_groups, 1, -1, hidden, at<uint8_t>(ws, L.qh),
                                      at<float>(ws, L.sh), Rt, nullptr, nullptr, nullptr, 0, h, g.max_total_rows,
                                      terms, status, st);
  };
  if (terms && !a_quantized && (err = quant_up(up)) != cudaSuccess) return MOE_ERR_CUDA;
  if (!record(events, 3, st)) return MOE_ERR_CUDA;
  if ((err = run(up)) != cudaSuccess) return MOE_ERR_CUDA;
  if (!record(events, 4, st)) return MOE_ERR_CUDA;
  if (terms && (err = quant_down(down)) != cudaSuccess) return MOE_ERR_CUDA;
  if (!record(events, 5, st)) return MOE_ERR_CUDA;
  if ((err = run(down)) != cudaSuccess) return MOE_ERR_CUDA;
  if (!record(events, 6, st)) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status reroute_impl(const moe_desc& d, int32_t* topk_idx, float* topk_w, const int32_t* counts,
                        const int32_t* row_of_slot, void* ws, cudaStream_t st) {
  const Layout L = make_layout(d);
  int32_t* changed = at<int32_t>(ws, L.rr_changed);
  RerouteScratch scratch{at<int32_t>(ws, L.rr_ex),      at<int8_t>(ws, L.rr_pick8), at<int32_t>(ws, L.rr_exl),
                         at<int32_t>(ws, L.rr_excount), at<int32_t>(ws, L.rr_claim), at<int32_t>(ws, L.rr_list)};
  cudaError_t e = launch_reroute_assign(d.num_tokens, d.num_experts, d.top_k, d.capacity, topk_idx,
                                        at<float>(ws, L.rr_key), counts, row_of_slot, scratch, changed,
                                        at<StatusBlock>(ws, L.status), st);
  if (e == cudaSuccess)
    e = launch_reroute_gates(d.num_tokens, d.num_experts, d.top_k, d.score_fn, d.renormalize,
                             at<float>(ws, L.rr_score), changed, topk_idx, topk_w, st);
  return cuda_status(e);
}

moe_status combine_impl(const moe_desc& d, const void* y_perm, const int32_t* row_of_slot, const float* topk_w,
                        void* y, cudaStream_t st, StatusBlock* status = nullptr) {
  CombineArgs a{};
  a.num_rows = routed_rows(d) + static_cast<int64_t>(d.num_shared) * d.num_tokens;
  a.status = status;
  a.S = d.num_tokens;
  a.d = d.d_model;
  a.K = d.top_k;
  a.act_dtype = d.act_dtype;
  a.y_perm = y_perm;
  a.row_of_slot = row_of_slot;
  a.topk_w = topk_w;
  a.shared_row0 = d.num_shared ? routed_rows(d) : -1;
  a.y = y;
  return cuda_status(launch_combine(a, st));
}

bool weights_ok(const moe_desc& d, const moe_weights* w) {
  if (w == nullptr) return false;
  if (d.act_dtype == MOE_F32 || d.activation == MOE_ACT_GELU) {
    if (!w->w1 || !w->w2 || !w->b1 || !w->b2) return false;
  } else {
    if (!w->w_gate || !w->w_up || !w->w_down) return false;
    if (d.weight_dtype == MOE_E4M3 && (!w->s_gate || !w->s_up || !w->s_down)) return false;
  }
  const void* ps[] = {w->w1, w->w2, w->w_gate, w->w_up, w->w_down};
  for (const void* p : ps)
    if (p && !aligned16(p)) return false;
  return true;
}

// The layer call (moe_layer_forward), recording the stage events of
// moe_layer_forward_timed when `events` is given.
moe_status layer_impl(const moe_desc* desc, const moe_weights* w, const void* x, void* y, int32_t* topk_idx,
                      float* topk_w, int32_t* counts, void* ws, size_t ws_bytes, void* stream, void* const* events) {
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  const moe_desc& d = *desc;
  if (d.num_tokens == 0) return MOE_OK;
  if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (!weights_ok(d, w) || w->w_router == nullptr || !aligned16(w->w_router)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout L = make_layout(d);
  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.topk_idx);
  float* gates = topk_w ? topk_w : at<float>(ws, L.topk_w);
  int32_t* cnt = counts ? counts : at<int32_t>(ws, L.counts);
  int32_t* offs = at<int32_t>(ws, L.offsets);
  int32_t* ros = at<int32_t>(ws, L.row_of_slot);
  int32_t* tor = at<int32_t>(ws, L.token_of_row);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  if (!record(events, 0, st)) return MOE_ERR_CUDA;
  const int terms = a_terms(d);
  if ((s = route_impl(d, w, x, nullptr, idx, gates, ws, st)) != MOE_OK) return s;
  if (d.reroute == 1) {
    // capacity ranks of the first choices, then the excess slots move; the
    // permutation below is that of the final choices
    if ((s = permute_impl(d, nullptr, idx, cnt, offs, ros, tor, nullptr, ws, st)) != MOE_OK) return s;
    if ((s = reroute_impl(d, idx, gates, cnt, ros, ws, st)) != MOE_OK) return s;
  }
  if (!record(events, 1, st)) return MOE_ERR_CUDA;
  // the permutation also writes the GEMM group tables, so the FFN skips that launch
  if (terms) {
    // E4M3 A rows: the row gather writes the codes and row scales straight
    // away (no bf16 copy of the permuted rows)
    if ((s = permute_impl(d, nullptr, idx, cnt, offs, ros, tor, nullptr, ws, st, true)) != MOE_OK) return s;
    const bool sh = d.num_shared != 0;
    if (launch_gather_quantize(d.num_tokens, d.d_model, d.top_k, ros, x, at<uint8_t>(ws, L.qa), at<float>(ws, L.sa),
                               sh ? at<uint8_t>(ws, L.qas) : nullptr, sh ? at<float>(ws, L.sas) : nullptr, terms,
                               st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (!record(events, 2, st)) return MOE_ERR_CUDA;
    if ((s = ffn_impl(d, *w, x_perm, offs, x, y_perm, ws, st, true, true, events)) != MOE_OK) return s;
  } else {
    if ((s = permute_impl(d, x, idx, cnt, offs, ros, tor, x_perm, ws, st, true)) != MOE_OK) return s;
    if (!record(events, 2, st)) return MOE_ERR_CUDA;
    if ((s = ffn_impl(d, *w, x_perm, offs, x, y_perm, ws, st, true, false, events)) != MOE_OK) return s;
  }
  if ((s = combine_impl(d, y_perm, ros, gates, y, st, at<StatusBlock>(ws, L.status))) != MOE_OK) return s;
  return record(events, 7, st) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

int64_t moe_routed_rows(const moe_desc* desc) {
  if (validate(desc) != MOE_OK) return -1;
  return routed_rows(*desc);
}

moe_status moe_workspace_size(const moe_desc* desc, size_t* bytes) {
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(*desc).total;
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < kAlign || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, kAlign, static_cast<cudaStream_t>(stream)));
}

moe_status moe_route(const moe_desc* desc, const moe_weights* w, const void* x, const float* logits_in,
                     int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_route");
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  if (desc->num_tokens == 0) return MOE_OK;
  if (topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (logits_in == nullptr) {
    if (x == nullptr || w == nullptr || w->w_router == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w->w_router)) return MOE_ERR_INVALID_ARG;
  }
  return route_impl(*desc, w, x, logits_in, topk_idx, topk_w, ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_permute(const moe_desc* desc, const void* x, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* row_of_slot, int32_t* token_of_row, void* x_perm, void* ws,
                       size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_permute");
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  if (counts == nullptr || offsets == nullptr || row_of_slot == nullptr || token_of_row == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (desc->num_tokens > 0 && topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (x && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  return permute_impl(*desc, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm, ws,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_grouped_ffn(const moe_desc* desc, const moe_weights* w, const void* x_perm, const int32_t* offsets,
                           const void* x, void* y_perm, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_grouped_ffn");
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  if (desc->num_tokens == 0) return MOE_OK;
  if (!weights_ok(*desc, w) || x_perm == nullptr || offsets == nullptr || y_perm == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (desc->num_shared && x == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(y_perm) || (x && !aligned16(x))) return MOE_ERR_INVALID_ARG;
  return ffn_impl(*desc, *w, x_perm, offsets, x, y_perm, ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_reroute(const moe_desc* desc, int32_t* topk_idx, float* topk_w, const int32_t* counts,
                       const int32_t* row_of_slot, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_reroute");
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if (desc->reroute != 1) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  if (desc->num_tokens == 0) return MOE_OK;
  if (topk_idx == nullptr || topk_w == nullptr || counts == nullptr || row_of_slot == nullptr)
    return MOE_ERR_INVALID_ARG;
  return reroute_impl(*desc, topk_idx, topk_w, counts, row_of_slot, ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_quantize_rows_e4m3(const void* x, int64_t rows, int32_t d, uint8_t* q, float* s, void* stream) {
  NvtxRange nvtx("moe_quantize_rows_e4m3");
  if (rows < 0 || d <= 0 || d % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (x == nullptr || q == nullptr || s == nullptr || !aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(s) & 3) != 0) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_rows(x, q, s, rows, d, 1, static_cast<cudaStream_t>(stream)));
}

moe_status moe_split_rows_e4m3(const void* x, int64_t rows, int32_t d, uint8_t* q, float* s, void* stream) {
  NvtxRange nvtx("moe_split_rows_e4m3");
  if (rows < 0 || d <= 0 || d % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (x == nullptr || q == nullptr || s == nullptr || !aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(s) & 3) != 0) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_rows(x, q, s, rows, d, 2, static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_desc* desc, const void* y_perm, const int32_t* row_of_slot, const float* topk_w,
                       void* y, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_combine");
  moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if ((s = check_ws(*desc, ws, ws_bytes)) != MOE_OK) return s;
  if (desc->num_tokens == 0) return MOE_OK;
  if (y_perm == nullptr || row_of_slot == nullptr || topk_w == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return combine_impl(*desc, y_perm, row_of_slot, topk_w, y, static_cast<cudaStream_t>(stream),
                      at<StatusBlock>(ws, make_layout(*desc).status));
}

moe_status moe_layer_forward(const moe_desc* desc, const moe_weights* w, const void* x, void* y, int32_t* topk_idx,
                             float* topk_w, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("moe_layer_forward");
  return layer_impl(desc, w, x, y, topk_idx, topk_w, counts, ws, ws_bytes, stream, nullptr);
}

moe_status moe_layer_forward_timed(const moe_desc* desc, const moe_weights* w, const void* x, void* y,
                                   int32_t* topk_idx, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                   void* stream, void* const* events) {
  NvtxRange nvtx("moe_layer_forward_timed");
  return layer_impl(desc, w, x, y, topk_idx, topk_w, counts, ws, ws_bytes, stream, events);
}

moe_status moe_load_stats(const moe_desc* desc, const int32_t* counts, double* stats, void* stream) {
  NvtxRange nvtx("moe_load_stats");
  const moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if (counts == nullptr || stats == nullptr || (reinterpret_cast<uintptr_t>(counts) & 3) != 0 ||
      (reinterpret_cast<uintptr_t>(stats) & 7) != 0)
    return MOE_ERR_INVALID_ARG;
  const int64_t slots = static_cast<int64_t>(desc->num_tokens) * desc->top_k;
  return cuda_status(launch_load_stats(desc->num_experts, slots, desc->capacity, counts, stats,
                                       static_cast<cudaStream_t>(stream)));
}

moe_status moe_bias_state_size(const moe_desc* desc, int32_t window_tokens, size_t* bytes) {
  const moe_status s = validate(desc);
  if (s != MOE_OK) return s;
  if (bytes == nullptr || window_tokens < 1) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(window_tokens) * desc->top_k > (int64_t(1) << 31) - 1) return MOE_ERR_INVALID_ARG;
  *bytes = bias_state_bytes(desc->num_experts, desc->top_k, window_tokens);
  return MOE_OK;
}

moe_status moe_bias_state_init(void* state, size_t state_bytes, void* stream) {
  if (state == nullptr || state_bytes < kAlign || (reinterpret_cast<uintptr_t>(state) & (kAlign - 1)) != 0)
    return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(state, 0, state_bytes, static_cast<cudaStream_t>(stream)));
}

moe_status moe_update_sel_bias(const moe_desc* desc, const int32_t* topk_idx, int32_t window_tokens, float gamma,
                               void* state, size_t state_bytes, float* sel_bias, int32_t* window_counts,
                               void* stream) {
  NvtxRange nvtx("moe_update_sel_bias");
  size_t need = 0;
  moe_status s = moe_bias_state_size(desc, window_tokens, &need);
  if (s != MOE_OK) return s;
  if (state == nullptr || state_bytes < need || (reinterpret_cast<uintptr_t>(state) & (kAlign - 1)) != 0)
    return MOE_ERR_WORKSPACE;
  if (sel_bias == nullptr || (desc->num_tokens > 0 && topk_idx == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!(gamma >= 0.0f) || gamma > 3.0e38f) return MOE_ERR_INVALID_ARG;  // also rejects NaN
  if (desc->num_tokens == 0) return MOE_OK;
  return cuda_status(launch_bias_update(desc->num_tokens, desc->num_experts, desc->top_k, window_tokens, topk_idx,
                                        gamma, state, sel_bias, window_counts, static_cast<cudaStream_t>(stream)));
}

moe_status moe_get_status(const void* ws, void* stream, uint32_t* flags, int32_t* counters) {
  if (ws == nullptr) return MOE_ERR_WORKSPACE;
  StatusBlock host;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&host, ws, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (flags) *flags = host.flags;
  if (counters) memcpy(counters, host.counters, sizeof(host.counters));
  const uint32_t errors = MOE_STATUS_NONFINITE_LOGIT | MOE_STATUS_BAD_EXPERT_ID | MOE_STATUS_TIMEOUT |
                          MOE_STATUS_BAD_GROUP | MOE_STATUS_DEBUG_CHECK;
  return (host.flags & errors) ? MOE_ERR_DEVICE_STATUS : MOE_OK;
}

const char* moe_strerror(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported combination";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_STATUS: return "device reported a data error (see moe_get_status)";
  }
  return "unknown status";
}

}  // extern "C"
