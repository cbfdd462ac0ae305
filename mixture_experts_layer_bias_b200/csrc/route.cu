// Router: logits, scoring and top-k selection.
//
// jsqmd.com "第11章 MoE模型推理" 11.1.1: R(x) = Softmax(W_r x) with the TopK
// sparsifier (non-selected scores set to -inf before the softmax, so the K
// gates are the softmax of the selected logits); 11.3.1 step 2 (top-k of the
// softmax probabilities, not renormalised).  ybb.press "MoE 推理工程深层实战"
// 2.3: aux-loss-free selection bias and group (node) limited selection: group
// score = sum of the group's biased scores, keep the best groups, pick the K
// experts inside them.  plumephp.com "MoE 混合专家推理", routing worked
// example: top-2 of the router's probabilities, outputs weighted by them.
//
// One warp routes one token.  Lane j holds experts j, 32+j, 64+j, ... in
// registers; group sums, the group choice and the K rounds of arg-max are warp
// shuffles.  Ties go to the lower expert (group) index; a NaN key ranks as
// -inf.  The selection-time sigmoid is computed with a fixed sequence of
// float32 operations so that its bits do not depend on the math library.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "pdl.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// exp(z) in float32 by Cody-Waite range reduction and the degree-7 Taylor
// polynomial, each step one IEEE float32 operation with round-to-nearest:
//   n = rint(z * log2 e), r = (z - n * ln2_hi) - n * ln2_lo,
//   p = 1 + r (1 + r (1/2! + r (1/3! + ... + r / 7!))), result = p * 2^n.
// ln2_hi is ln 2 truncated to 16 significant bits (so n * ln2_hi is exact for
// |n| < 256) and ln2_lo the float32 rounding of the remainder; the Taylor
// coefficients are the float32 roundings of 1/j!.  z > 88 gives +inf and
// z < -30 gives 0 (there 1 + exp(z) rounds to 1 anyway).
__device__ __forceinline__ float exp_cw_f32(float z) {
  if (z > 88.0f) return __int_as_float(0x7f800000);
  if (z < -30.0f) return 0.0f;
  const float kLog2e = __int_as_float(0x3fb8aa3b);   // 1/ln 2
  const float kLn2Hi = __int_as_float(0x3f317200);   // 0.693145751953125
  const float kLn2Lo = __int_as_float(0x35bfbe8e);   // ln 2 - kLn2Hi
  const float n = rintf(__fmul_rn(z, kLog2e));
  float r = __fsub_rn(z, __fmul_rn(n, kLn2Hi));
  r = __fsub_rn(r, __fmul_rn(n, kLn2Lo));
  float p = __int_as_float(0x39500d01);                  // 1/7!
  p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3ab60b61));  // 1/6!
  p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3c088889));  // 1/5!
  p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3d2aaaab));  // 1/4!
  p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3e2aaaab));  // 1/3!
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);                        // 1/2!
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);                        // 1/1!
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);                        // 1/0!
  return ldexpf(p, static_cast<int>(n));
}

// sigma(l) = 1 / (1 + exp(-l)) with the exponential above.
__device__ __forceinline__ float sigmoid_sel_f32(float l) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cw_f32(-l)));
}

__device__ __forceinline__ void warp_argmax(float& v, int& idx) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float ov = __shfl_xor_sync(kFull, v, off);
    const int oi = __shfl_xor_sync(kFull, idx, off);
    if (ov > v || (ov == v && oi < idx)) {
      v = ov;
      idx = oi;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

struct SelectParams {
  int E, K, score_fn, renormalize, num_groups, topk_groups;
  float tau;  // softmax temperature (1 = none): z = l / tau
  const float* sel_bias;
  int32_t* topk_idx;
  float* topk_w;
  StatusBlock* status;
  float* cand_key;   // optional [S][E]: selection key of each candidate expert, -inf for the others
  float* score_out;  // optional [S][E]: the gate source (logit, or sigmoid score) of every expert
};

// Gate of this lane's selected expert (lanes < K hold one each, my_score its
// score); score[]/valid[] are the token's scores of experts 32*i + lane.
template <int NI>
__device__ __forceinline__ float gate_of(const float (&score)[NI], const bool (&valid)[NI], float my_score,
                                         bool mine, int score_fn, int renormalize) {
  const float kNegInf = __int_as_float(0xff800000);
  if (score_fn == MOE_SCORE_SOFTMAX) {
    if (renormalize) {
      const float m = warp_max(mine ? my_score : kNegInf);
      const float ex = mine ? expf(my_score - m) : 0.0f;
      return ex / warp_sum(ex);
    }
    float m = kNegInf;
#pragma unroll
    for (int i = 0; i < NI; ++i)
      if (valid[i]) m = fmaxf(m, score[i]);
    m = warp_max(m);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i)
      if (valid[i]) s += expf(score[i] - m);
    s = warp_sum(s);
    return expf(my_score - m) / s;
  }
  if (renormalize) {
    const float s = warp_sum(mine ? my_score : 0.0f);
    return my_score / s;
  }
  return my_score;
}

// Selection for one token held by the whole warp: l[i] is the logit (router
// bias included) of expert 32*i + lane.  Writes K indices and gates.
// Softmax scores are the logits divided by the temperature (jsqmd.com
// 11.3.3, soft routing with softmax(s / tau)).
template <int NI>
__device__ void select_topk(const float (&l)[NI], const SelectParams& p, int t) {
  const int lane = lane_id();
  const int E = p.E;
  const float kNegInf = __int_as_float(0xff800000);
  float score[NI], key[NI];
  bool valid[NI], cand[NI], taken[NI];
  bool nonfinite = false;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int e = 32 * i + lane;
    valid[i] = e < E;
    const float li = valid[i] ? l[i] : kNegInf;
    if (valid[i] && !isfinite(li)) nonfinite = true;
    // softmax: the tempered logit z = l / tau (one float32 division, exact for
    // tau = 1) is both the gate source and the key; sigmoid: sigma(l)
    score[i] = (p.score_fn == MOE_SCORE_SIGMOID) ? sigmoid_sel_f32(li) : __fdiv_rn(li, p.tau);
    float k = score[i];
    if (valid[i] && p.sel_bias != nullptr) k = __fadd_rn(k, __ldg(p.sel_bias + e));
    if (!valid[i] || isnan(k)) k = kNegInf;
    key[i] = k;
    cand[i] = valid[i];
    taken[i] = false;
  }
  if (__any_sync(kFull, nonfinite) && lane == 0) report(p.status, MOE_STATUS_NONFINITE_LOGIT, MOE_CNT_NONFINITE);

  if (p.num_groups > 1) {
    const int gs = E / p.num_groups;  // power of two
    float gsum[NI];
    if (gs >= 32) {
      // members of group g: registers g*r .. g*r + r - 1 in every lane.  The
      // halving tree first adds register j to register j + r/2 (member m to
      // m + gs/2), down to single registers, then goes across lanes.
      const int r = gs >> 5;
      float v[NI];
#pragma unroll
      for (int i = 0; i < NI; ++i) v[i] = key[i];
#pragma unroll
      for (int half = NI / 2; half >= 1; half >>= 1) {
        if (half < r) {
#pragma unroll
          for (int i = 0; i < NI; ++i)
            if (i + half < NI && (i % r) < half) v[i] = __fadd_rn(v[i], v[i + half]);
        }
      }
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        if (i % r == 0) {
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) v[i] = __fadd_rn(v[i], __shfl_xor_sync(kFull, v[i], off));
        }
      }
#pragma unroll
      for (int i = 0; i < NI; ++i) gsum[i] = v[(i / r) * r];
    } else {
      // gs consecutive lanes form a group: butterfly inside the group
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        float v = key[i];
        for (int off = gs >> 1; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, off));
        gsum[i] = v;
      }
    }
    bool gchosen[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      if (isnan(gsum[i])) gsum[i] = kNegInf;
      gchosen[i] = false;
    }
    for (int rnd = 0; rnd < p.topk_groups; ++rnd) {
      float bv = kNegInf;
      int bg = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int gid = (32 * i + lane) / gs;
        if (valid[i] && !gchosen[i] && (gsum[i] > bv || (gsum[i] == bv && gid < bg))) {
          bv = gsum[i];
          bg = gid;
        }
      }
      warp_argmax(bv, bg);
#pragma unroll
      for (int i = 0; i < NI; ++i)
        if ((32 * i + lane) / gs == bg) gchosen[i] = true;
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) cand[i] = cand[i] && gchosen[i];
  }
  if (p.cand_key != nullptr) {
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int e = 32 * i + lane;
      if (valid[i]) {
        p.cand_key[static_cast<int64_t>(t) * E + e] = cand[i] ? key[i] : kNegInf;
        p.score_out[static_cast<int64_t>(t) * E + e] = score[i];
      }
    }
  }

  int my_e = 0;
  float my_score = 0.0f;
  for (int k = 0; k < p.K; ++k) {
    float bv = kNegInf;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int e = 32 * i + lane;
      if (cand[i] && !taken[i] && (key[i] > bv || (key[i] == bv && e < be))) {
        bv = key[i];
        be = e;
      }
    }
    warp_argmax(bv, be);
    float sc = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      if (32 * i + lane == be) {
        taken[i] = true;
        sc = score[i];
      }
    }
    sc = __shfl_sync(kFull, sc, be & 31);
    if (lane == k) {
      my_e = be;
      my_score = sc;
    }
  }

  const bool mine = lane < p.K;
  const float g = gate_of<NI>(score, valid, my_score, mine, p.score_fn, p.renormalize);
  if (mine) {
    p.topk_idx[static_cast<int64_t>(t) * p.K + lane] = my_e;
    p.topk_w[static_cast<int64_t>(t) * p.K + lane] = g;
  }
}

constexpr int kRouteWarps = 8;

// E <= EMAX <= 32: the warp computes the token's logits itself.  Lanes stride
// over 16-byte vectors of x and W_r rows (fp32 partial sums), then a butterfly
// reduction per expert.
template <typename T, int EMAX>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_fused_kernel(int S, int d, const T* __restrict__ x, const T* __restrict__ w_router,
                       const float* __restrict__ router_bias, SelectParams p) {
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= S) return;
  const int lane = lane_id();
  constexpr int V = Vec16<T>::N;
  const int nvec = d / V;
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.0f;
  const T* xr = x + static_cast<int64_t>(t) * d;
  for (int v = lane; v < nvec; v += 32) {
    float xf[V];
    unpack16<T>(ldg16(xr + v * V), xf);
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < p.E) {
        float wf[V];
        unpack16<T>(ldg16(w_router + static_cast<int64_t>(e) * d + v * V), wf);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[e] = fmaf(xf[j], wf[j], acc[e]);
      }
    }
  }
  float l[1] = {0.0f};
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    const float s = warp_sum(acc[e]);
    if (e == lane) l[0] = s;
  }
  if (lane < p.E && router_bias != nullptr) l[0] = __fadd_rn(l[0], __ldg(router_bias + lane));
  select_topk<1>(l, p, t);
}

// Small batches (decode): one CTA per token, its 8 warps split d so the
// token's dot products are not serialised on one warp.  Per-warp partial sums
// are added in warp order (deterministic), then warp 0 selects.
template <typename T, int EMAX>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_token_cta_kernel(int d, const T* __restrict__ x, const T* __restrict__ w_router,
                           const float* __restrict__ router_bias, SelectParams p) {
  __shared__ float part[kRouteWarps][EMAX];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = lane_id();
  constexpr int V = Vec16<T>::N;
  const int nvec = d / V;
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.0f;
  const T* xr = x + static_cast<int64_t>(t) * d;
  for (int v = threadIdx.x; v < nvec; v += kRouteWarps * 32) {
    float xf[V];
    unpack16<T>(ldg16(xr + v * V), xf);
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < p.E) {
        float wf[V];
        unpack16<T>(ldg16(w_router + static_cast<int64_t>(e) * d + v * V), wf);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[e] = fmaf(xf[j], wf[j], acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    const float s = warp_sum(acc[e]);
    if (lane == 0) part[warp][e] = s;
  }
  __syncthreads();
  if (warp != 0) return;
  float l[1] = {0.0f};
  if (lane < p.E && lane < EMAX) {
    float s = 0.0f;
    for (int w = 0; w < kRouteWarps; ++w) s += part[w][lane];
    l[0] = router_bias != nullptr ? __fadd_rn(s, __ldg(router_bias + lane)) : s;
  }
  select_topk<1>(l, p, t);
}

// Logits given in memory (caller-supplied, or computed by the logits kernel).
template <int NI>
__global__ void __launch_bounds__(kRouteWarps * 32)
    topk_kernel(int S, const float* __restrict__ logits, const float* __restrict__ router_bias, SelectParams p) {
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= S) return;
  const int lane = lane_id();
  float l[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int e = 32 * i + lane;
    float v = 0.0f;
    if (e < p.E) {
      v = __ldg(logits + static_cast<int64_t>(t) * p.E + e);
      if (router_bias != nullptr) v = __fadd_rn(v, __ldg(router_bias + e));
    }
    l[i] = v;
  }
  select_topk<NI>(l, p, t);
}

// Plain tiled SIMT GEMM for the router logits when E > 32: out[t][e] =
// sum_k x[t][k] * W_r[e][k] in fp32.  Tile 32 tokens x 64 experts, K-chunks
// of 32 staged in shared memory.
template <typename T>
__global__ void __launch_bounds__(256)
    logits_kernel(int S, int d, int E, const T* __restrict__ x, const T* __restrict__ w, float* __restrict__ out) {
  __shared__ float xs[32][33];
  __shared__ float ws[64][33];
  const int t0 = blockIdx.x * 32, e0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;  // 16 x 16 threads: 2 tokens x 4 experts each
  float acc[2][4] = {};
  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int i = tid; i < 32 * 32; i += 256) {
      const int r = i >> 5, c = i & 31;
      xs[r][c] = (t0 + r < S && k0 + c < d) ? to_f32<T>(x[static_cast<int64_t>(t0 + r) * d + k0 + c]) : 0.0f;
    }
    for (int i = tid; i < 64 * 32; i += 256) {
      const int r = i >> 5, c = i & 31;
      ws[r][c] = (e0 + r < E && k0 + c < d) ? to_f32<T>(w[static_cast<int64_t>(e0 + r) * d + k0 + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const float a0 = xs[ty * 2][c], a1 = xs[ty * 2 + 1][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float b = ws[tx * 4 + j][c];
        acc[0][j] = fmaf(a0, b, acc[0][j]);
        acc[1][j] = fmaf(a1, b, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty * 2 + i, e = e0 + tx * 4 + j;
      if (t < S && e < E) out[static_cast<int64_t>(t) * E + e] = acc[i][j];
    }
}

// Gates of a token whose experts changed after selection (over-capacity
// re-routing): a warp per token, lanes holding the gate sources of experts
// 32*i + lane as in the selection, lanes < K one selected expert each.
template <int NI>
__global__ void __launch_bounds__(kRouteWarps * 32)
    reroute_gates_kernel(int S, int E, int K, int score_fn, int renormalize, const float* __restrict__ score_in,
                         const int32_t* __restrict__ changed, const int32_t* __restrict__ topk_idx,
                         float* __restrict__ topk_w) {
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= S || changed[t] == 0) return;
  const int lane = lane_id();
  const float* row = score_in + static_cast<int64_t>(t) * E;
  float score[NI];
  bool valid[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int e = 32 * i + lane;
    valid[i] = e < E;
    score[i] = valid[i] ? row[e] : __int_as_float(0xff800000);
  }
  const bool mine = lane < K;
  const int my_e = mine ? topk_idx[static_cast<int64_t>(t) * K + lane] : 0;
  const float my_score = (mine && my_e >= 0 && my_e < E) ? row[my_e] : 0.0f;
  const float g = gate_of<NI>(score, valid, my_score, mine, score_fn, renormalize);
  if (mine) topk_w[static_cast<int64_t>(t) * K + lane] = g;
}

template <int NI>
cudaError_t launch_topk_ni(const RouteArgs& a, const float* logits, const SelectParams& sp, cudaStream_t st) {
  const int blocks = (a.S + kRouteWarps - 1) / kRouteWarps;
  topk_kernel<NI><<<blocks, kRouteWarps * 32, 0, st>>>(a.S, logits, a.router_bias, sp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream) {
  if (a.S == 0) return cudaSuccess;
  SelectParams sp{a.E,        a.K,      a.score_fn, a.renormalize, a.num_groups,   a.topk_groups, a.tau,
                  a.sel_bias, a.topk_idx, a.topk_w, a.status,      a.cand_key_out, a.score_out};
  const int blocks = (a.S + kRouteWarps - 1) / kRouteWarps;
  const float* logits = a.logits;
  if (logits == nullptr && a.E <= 32) {
    // decode-sized batches: a CTA per token; otherwise a warp per token
    const bool per_cta = a.S <= 512;
    const int g = per_cta ? a.S : blocks;
    cudaError_t err = cudaSuccess;
#define MOE_ROUTE_LAUNCH(T, EM)                                                                                \
  do {                                                                                                         \
    if (per_cta)                                                                                               \
      err = launch_pdl(route_token_cta_kernel<T, EM>, dim3(g), dim3(kRouteWarps * 32), 0, stream, a.d,              \
                       static_cast<const T*>(a.x), static_cast<const T*>(a.w_router), a.router_bias, sp);      \
    else                                                                                                       \
      route_fused_kernel<T, EM><<<g, kRouteWarps * 32, 0, stream>>>(                                           \
          a.S, a.d, static_cast<const T*>(a.x), static_cast<const T*>(a.w_router), a.router_bias, sp);         \
  } while (0)
    if (a.act_dtype == MOE_BF16) {
      if (a.E <= 8)
        MOE_ROUTE_LAUNCH(__nv_bfloat16, 8);
      else
        MOE_ROUTE_LAUNCH(__nv_bfloat16, 32);
    } else {
      if (a.E <= 8)
        MOE_ROUTE_LAUNCH(float, 8);
      else
        MOE_ROUTE_LAUNCH(float, 32);
    }
#undef MOE_ROUTE_LAUNCH
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  if (logits == nullptr) {
    cudaError_t err;
    if (a.act_dtype == MOE_BF16 && a.d % 8 == 0) {
      // l = x W_r^T as one dense GEMM on the tensor cores (fp32 accumulate
      // and output); the selection then reads the logits back
      GemmArgs g{};
      g.epilogue = EPI_NONE;
      g.groups = nullptr;
      g.num_groups = 1;
      g.shared_slab = -1;
      g.a = a.x;
      g.a_rows = a.S;
      g.b0 = a.w_router;
      g.b_rows = a.E;
      g.n_per_slab = a.E;
      g.N = a.E;
      g.K = a.d;
      g.out = a.logits_scratch;
      g.out_rows = a.S;
      g.out_f32 = 1;
      g.max_total_rows = a.S;
      g.max_group_rows = a.S;
      g.status = a.status;
      err = launch_grouped_gemm_tc(g, a.num_sms, stream);
    } else {
      dim3 grid((a.S + 31) / 32, (a.E + 63) / 64);
      if (a.act_dtype == MOE_BF16)
        logits_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a.S, a.d, a.E, static_cast<const __nv_bfloat16*>(a.x),
                                                                static_cast<const __nv_bfloat16*>(a.w_router),
                                                                a.logits_scratch);
      else
        logits_kernel<float><<<grid, 256, 0, stream>>>(a.S, a.d, a.E, static_cast<const float*>(a.x),
                                                        static_cast<const float*>(a.w_router), a.logits_scratch);
      err = cudaGetLastError();
    }
    if (err != cudaSuccess) return err;
    logits = a.logits_scratch;
  }
  const int ni = (a.E + 31) / 32;
  if (ni <= 1) return launch_topk_ni<1>(a, logits, sp, stream);
  if (ni <= 2) return launch_topk_ni<2>(a, logits, sp, stream);
  if (ni <= 4) return launch_topk_ni<4>(a, logits, sp, stream);
  return launch_topk_ni<8>(a, logits, sp, stream);
}

cudaError_t launch_reroute_gates(int S, int E, int K, int score_fn, int renormalize, const float* score,
                                 const int32_t* changed, const int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  const int blocks = (S + kRouteWarps - 1) / kRouteWarps;
  const int ni = (E + 31) / 32;
#define MOE_RG(N) \
  reroute_gates_kernel<N><<<blocks, kRouteWarps * 32, 0, stream>>>(S, E, K, score_fn, renormalize, score, changed, \
                                                                   topk_idx, topk_w)
  if (ni <= 1)
    MOE_RG(1);
  else if (ni <= 2)
    MOE_RG(2);
  else if (ni <= 4)
    MOE_RG(4);
  else
    MOE_RG(8);
#undef MOE_RG
  return cudaGetLastError();
}

}  // namespace moe
