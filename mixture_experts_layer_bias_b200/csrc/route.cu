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
#include "route_select.cuh"

namespace moe {

namespace {

using namespace route_detail;

constexpr int kRouteWarps = 8;

// fp32 activations, E <= EMAX <= 32, large batches (bf16 rows take the
// tensor-core kernel below): every warp routes TPW tokens (2 for
// EMAX = 8, 1 for EMAX = 32) over the whole of d, lanes striding over 16-byte
// vectors; 8 (EMAX = 8) or 4 vectors of each token are loaded together per
// lane (a token row's loads in four rounds at d = 4096), so the
// token rows -- the bytes that must come from HBM -- stream with many loads in
// flight and no block-wide barrier.  The router weights sit in shared memory
// (at most 64 KB: larger router matrices go through the logits GEMM, see
// route_logits_first).  The TPW x EMAX
// partial dot products of a lane are summed over the warp by a reduce-scatter
// butterfly (lane i ends with value i: token i / EMAX, expert i % EMAX), then
// the warp selects its tokens.  The grid is persistent: warps loop over token
// sets.
constexpr int kRouteRowWarps = 8;

template <typename T, int EMAX>
__global__ void __launch_bounds__(kRouteRowWarps * 32, 2)
    route_rows_kernel(int S, int d, const T* __restrict__ x, const T* __restrict__ w_router,
                      const float* __restrict__ router_bias, SelectParams p) {
  constexpr int TPW = EMAX >= 16 ? 1 : 16 / EMAX;
  constexpr int NV = TPW * EMAX;  // 16 or 32 partial sums per lane
  constexpr int kRouteBatch = EMAX >= 16 ? 4 : 8;
  constexpr int V = Vec16<T>::N;
  extern __shared__ uint4 wsm[];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int nvec = d / V;
  {
    const int n16 = p.E * nvec;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) wsm[i] = ldg16(w_router + static_cast<int64_t>(i) * V);
    __syncthreads();
  }
  const float bias = (lane < p.E && router_bias != nullptr) ? __ldg(router_bias + lane) : 0.0f;
  const int num_sets = (S + TPW - 1) / TPW;
  for (int set = blockIdx.x * kRouteRowWarps + warp; set < num_sets; set += gridDim.x * kRouteRowWarps) {
    const int t0 = set * TPW;
    const T* xr[TPW];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) xr[tt] = x + static_cast<int64_t>(min(t0 + tt, S - 1)) * d;
    float acc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] = 0.0f;
    for (int vb = lane; vb < nvec; vb += 32 * kRouteBatch) {
      uint4 xv[TPW][kRouteBatch];
#pragma unroll
      for (int b = 0; b < kRouteBatch; ++b)
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
          xv[tt][b] = (vb + 32 * b < nvec) ? ldg16(xr[tt] + (vb + 32 * b) * V) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int b = 0; b < kRouteBatch; ++b) {
        const int v = vb + 32 * b;
        if (v >= nvec) break;
        float xf[TPW][V];
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) unpack16<T>(xv[tt][b], xf[tt]);
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < p.E) {
            float wf[V];
            unpack16<T>(wsm[e * nvec + v], wf);
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
              for (int j = 0; j < V; ++j) acc[tt * EMAX + e] = fmaf(xf[tt][j], wf[j], acc[tt * EMAX + e]);
          }
        }
      }
    }
    // reduce-scatter over the warp: afterwards acc[0] of lane i is the warp's sum of value i % NV
#pragma unroll
    for (int s = NV / 2; s >= 1; s >>= 1) {
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int i = 0; i < s; ++i) {
        const float send = upper ? acc[i] : acc[i + s];
        const float keep = upper ? acc[i + s] : acc[i];
        acc[i] = keep + __shfl_xor_sync(kFull, send, s);
      }
    }
#pragma unroll
    for (int s = NV; s < 32; s <<= 1) acc[0] += __shfl_xor_sync(kFull, acc[0], s);
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      if (t0 + tt >= S) break;  // warp-uniform
      float l[1];
      l[0] = __shfl_sync(kFull, acc[0], tt * EMAX + (lane % EMAX));
      if (lane < p.E && router_bias != nullptr) l[0] = __fadd_rn(l[0], bias);
      select_topk<1>(l, p, t0 + tt);
    }
  }
}

// bf16, E <= EMAX <= 32, large batches: the logits of 16 tokens against 8
// experts over 16 columns of d are one m16n8k16 tensor-core product (bf16
// operands, fp32 accumulation), so streaming the token rows costs no
// per-element unpacking or FMA work and the pass is bound by reading x.  A
// CTA owns 16 tokens; its warps split d into 32-column chunks (warp w takes
// chunks w, w + 8, ...).  Per chunk, lane (g = lane / 4, q = lane % 4) loads
// the 16 bytes at column 32c + 8q of token rows g and g + 8 and of router row
// 8nt + g (L1/L2-resident): the quad's four lanes hold the chunk's 32
// columns, and since the A and B fragments give a lane the same fragment
// slots, columns 8q..8q+3 (8q+4..8q+7) fill slots {2q, 2q+1, 2q+8, 2q+9} of
// the chunk's first (second) product and every column is summed once.  The
// warps' partial logits are added in warp order through shared memory, then
// each warp selects two of the CTA's tokens.
constexpr int kRouteMmaWarps = 8;
constexpr int kRouteMmaTokens = 16;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte read-only loads kept in program order with the products (volatile
// asm), so a lane's U chunks are all in flight before the first product;
// token rows are read once and bypass L1, router rows stay in L1
__device__ __forceinline__ uint4 ld16_stream(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}
__device__ __forceinline__ uint4 ld16_keep(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

template <int EMAX>
__global__ void __launch_bounds__(kRouteMmaWarps * 32, 2)
    route_rows_mma_kernel(int S, int d, const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
                          const float* __restrict__ router_bias, SelectParams p) {
  constexpr int NT = EMAX / 8;                  // n-tiles of 8 experts
  constexpr int ACC = NT == 1 ? 2 : 1;          // independent accumulator chains per n-tile
  constexpr int U = NT == 1 ? 8 : 3;            // chunks in flight per lane
  __shared__ float part[kRouteMmaWarps][kRouteMmaTokens][EMAX];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int g = lane >> 2, q = lane & 3;
  const int t0 = blockIdx.x * kRouteMmaTokens;
  const __nv_bfloat16* xa = x + static_cast<int64_t>(min(t0 + g, S - 1)) * d;
  const __nv_bfloat16* xb = x + static_cast<int64_t>(min(t0 + g + 8, S - 1)) * d;
  const __nv_bfloat16* wr[NT];
  bool wok[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = nt * 8 + g;
    wok[nt] = n < p.E;
    wr[nt] = w + static_cast<int64_t>(wok[nt] ? n : 0) * d;
  }
  float acc[ACC][NT][4];
#pragma unroll
  for (int s = 0; s < ACC; ++s)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[s][nt][i] = 0.0f;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  // full chunks, U per lane at a time: unconditional loads (rows of absent
  // experts read router row 0 and are zeroed after the load)
  const int nfull = d / 32;
  int c0 = warp;
  for (; c0 + (U - 1) * kRouteMmaWarps < nfull; c0 += kRouteMmaWarps * U) {
    uint4 va[U], vb[U], vw[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int col = (c0 + u * kRouteMmaWarps) * 32 + q * 8;
      va[u] = ld16_stream(xa + col);
      vb[u] = ld16_stream(xb + col);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4 v = ld16_keep(wr[nt] + col);
        vw[u][nt] = wok[nt] ? v : zero;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float(&c)[4] = acc[u % ACC][nt];
        mma_bf16_16816(c, va[u].x, vb[u].x, va[u].y, vb[u].y, vw[u][nt].x, vw[u][nt].y);
        mma_bf16_16816(c, va[u].z, vb[u].z, va[u].w, vb[u].w, vw[u][nt].z, vw[u][nt].w);
      }
  }
  // the remaining chunks one at a time; the last may be partial (d % 8 == 0:
  // a lane's 8 columns are all inside d or all outside)
  const int nch = (d + 31) / 32;
  for (; c0 < nch; c0 += kRouteMmaWarps) {
    const int col = c0 * 32 + q * 8;
    const bool ok = col < d;
    const uint4 va = ok ? ldg16(xa + col) : zero;
    const uint4 vb = ok ? ldg16(xb + col) : zero;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 vw = (ok && wok[nt]) ? ldg16(wr[nt] + col) : zero;
      mma_bf16_16816(acc[0][nt], va.x, vb.x, va.y, vb.y, vw.x, vw.y);
      mma_bf16_16816(acc[0][nt], va.z, vb.z, va.w, vb.w, vw.z, vw.w);
    }
  }
  // C fragment: c0, c1 = token g, experts 8nt + 2q + {0, 1}; c2, c3 = token g + 8
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = ACC == 2 ? acc[0][nt][i] + acc[ACC - 1][nt][i] : acc[0][nt][i];
    const int n = nt * 8 + 2 * q;
    part[warp][g][n] = c[0];
    part[warp][g][n + 1] = c[1];
    part[warp][g + 8][n] = c[2];
    part[warp][g + 8][n + 1] = c[3];
  }
  __syncthreads();
  const float bias = (lane < p.E && router_bias != nullptr) ? __ldg(router_bias + lane) : 0.0f;
#pragma unroll
  for (int i = 0; i < kRouteMmaTokens / kRouteMmaWarps; ++i) {
    const int tl = warp * (kRouteMmaTokens / kRouteMmaWarps) + i;
    if (t0 + tl >= S) break;  // warp-uniform
    float l[1] = {0.0f};
    if (lane < EMAX) {
      float s = 0.0f;
#pragma unroll
      for (int w2 = 0; w2 < kRouteMmaWarps; ++w2) s += part[w2][tl][lane];
      l[0] = (lane < p.E && router_bias != nullptr) ? __fadd_rn(s, bias) : s;
    }
    select_topk<1>(l, p, t0 + tl);
  }
}

// Small batches (decode): one CTA per token, its 16 warps split d (d = 4096
// in bf16 is one 16-byte vector per thread, so every load of the token is in
// flight at once).  Per-warp partial sums are added in warp order
// (deterministic), then warp 0 selects.
constexpr int kRouteTokenWarps = 16;

template <typename T, int EMAX>
__global__ void __launch_bounds__(kRouteTokenWarps * 32)
    route_token_cta_kernel(int d, const T* __restrict__ x, const T* __restrict__ w_router,
                           const float* __restrict__ router_bias, SelectParams p) {
  __shared__ float part[kRouteTokenWarps][EMAX];
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
  for (int v = threadIdx.x; v < nvec; v += kRouteTokenWarps * 32) {
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
    for (int w = 0; w < kRouteTokenWarps; ++w) s += part[w][lane];
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

template <typename T, int EM>
cudaError_t launch_route_token_cta(const RouteArgs& a, const SelectParams& sp, cudaStream_t st) {
  return launch_pdl(route_token_cta_kernel<T, EM>, dim3(a.S), dim3(kRouteTokenWarps * 32), 0, st, a.d,
                    static_cast<const T*>(a.x), static_cast<const T*>(a.w_router), a.router_bias, sp);
}

template <int EM>
cudaError_t launch_route_rows_mma(const RouteArgs& a, const SelectParams& sp, cudaStream_t st) {
  const dim3 grid((a.S + kRouteMmaTokens - 1) / kRouteMmaTokens);
  route_rows_mma_kernel<EM><<<grid, kRouteMmaWarps * 32, 0, st>>>(a.S, a.d, static_cast<const __nv_bfloat16*>(a.x),
                                                                   static_cast<const __nv_bfloat16*>(a.w_router),
                                                                   a.router_bias, sp);
  return cudaGetLastError();
}

template <int EM>
cudaError_t launch_route_rows_f32(const RouteArgs& a, const SelectParams& sp, cudaStream_t st) {
  constexpr int TPW = EM >= 16 ? 1 : 16 / EM;
  const int sets = (a.S + TPW - 1) / TPW;
  const int want = (sets + kRouteRowWarps - 1) / kRouteRowWarps;
  const int cap = (a.num_sms > 0 ? a.num_sms : 148) * 2;
  const int grid = want < cap ? want : cap;
  const size_t wbytes = static_cast<size_t>(a.E) * a.d * sizeof(float);  // <= kRouteWSmemBytes here
  cudaError_t err =
      cudaFuncSetAttribute(route_rows_kernel<float, EM>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouteWSmemBytes);
  if (err != cudaSuccess) return err;
  route_rows_kernel<float, EM><<<grid, kRouteRowWarps * 32, wbytes, st>>>(
      a.S, a.d, static_cast<const float*>(a.x), static_cast<const float*>(a.w_router), a.router_bias, sp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream) {
  if (a.S == 0) return cudaSuccess;
  SelectParams sp{a.E,        a.K,      a.score_fn, a.renormalize, a.num_groups,   a.topk_groups, a.tau,
                  a.sel_bias, a.topk_idx, a.topk_w, a.status,      a.cand_key_out, a.score_out};
  const float* logits = a.logits;
  const int elem = a.act_dtype == MOE_F32 ? 4 : 2;
  if (logits == nullptr && !route_logits_first(a.S, a.E, a.d, elem)) {
    // decode-sized batches: a CTA per token; otherwise 16 tokens per CTA on
    // the tensor cores (bf16; d % 8 == 0 for every layer) or warps streaming
    // token rows (fp32)
    const bool per_cta = a.S <= 512;
    const bool wide = a.E > 8;
    cudaError_t err;
    if (a.act_dtype == MOE_BF16) {
      if (per_cta)
        err = wide ? launch_route_token_cta<__nv_bfloat16, 32>(a, sp, stream)
                   : launch_route_token_cta<__nv_bfloat16, 8>(a, sp, stream);
      else
        err = wide ? launch_route_rows_mma<32>(a, sp, stream) : launch_route_rows_mma<8>(a, sp, stream);
    } else {
      if (per_cta)
        err = wide ? launch_route_token_cta<float, 32>(a, sp, stream) : launch_route_token_cta<float, 8>(a, sp, stream);
      else
        err = wide ? launch_route_rows_f32<32>(a, sp, stream) : launch_route_rows_f32<8>(a, sp, stream);
    }
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
