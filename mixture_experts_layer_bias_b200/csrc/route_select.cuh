// Expert selection of one token held by one warp: scores (softmax logits
// with temperature, or the operationally defined sigmoid), selection bias,
// group-limited candidates, K rounds of arg-max and the gate weights.  Shared
// by the routing kernels.
//
// jsqmd.com "第11章 MoE模型推理" 11.1.1 (R(x) = Softmax(W_r x) with the TopK
// sparsifier), 11.3.3 (soft routing with a temperature); ybb.press
// "MoE 推理工程深层实战" 2.3 (aux-loss-free selection bias, group-limited
// selection).
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {
namespace route_detail {

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

}  // namespace route_detail
}  // namespace moe
