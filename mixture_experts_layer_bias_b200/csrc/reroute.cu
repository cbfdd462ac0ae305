// Over-capacity re-routing of excess slots to the next-best expert.
//
// jsqmd.com "第11章 MoE模型推理" 11.3.3 (expert-dropping paragraph): when an expert is
// overloaded, the tokens above its share are routed again to their next-best
// expert.  Reading taken (the page gives one sentence): every expert keeps its
// first C slots in (token, k) order -- the primary rows of the capacity-bounded
// permutation -- and the excess slots, in (token, k) order, each take the
// candidate expert with the highest selection key among those that still have
// room and that the token does not already hold (ties to the lower index);
// an excess slot with no such expert keeps its expert and its overflow row.
//
// The visit order makes this a serial assignment.  One CTA runs it in rounds
// over chunks of up to 1024 excess slots: every slot picks its expert against
// the room left at the start of the round (8 lanes per slot, splitting the
// experts; a token's slots in one chunk go to one lane group, in k order, each
// excluding the previous picks), the
// picks are ranked per expert in slot order, and the longest prefix of slots
// whose pick still fits is committed.  A pick made against the round's room
// is the serial pick as long as every earlier slot's pick fit (room only
// shrinks, and the picked expert is still available), so the committed prefix
// equals the serial result; the first slot that does not fit had filled its
// expert, so a chunk is cut short at most once per expert.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 256;
constexpr int kG = 8;                     // lanes per slot pick (kMaxE / kG <= 32 held bits)
constexpr int kSpan = kThreads / (kThreads / kG);  // slots per group and round (a chunk over all groups)

__global__ void __launch_bounds__(kThreads, 1)
    reroute_assign_kernel(int S, int E, int K, int C, int32_t* __restrict__ topk_idx,
                          const float* __restrict__ cand_key, const int32_t* __restrict__ counts,
                          const int32_t* __restrict__ row_of_slot, int32_t* __restrict__ ex,
                          int32_t* __restrict__ changed, StatusBlock* status) {
  __shared__ int room[kMaxE];
  __shared__ int wcnt[kWarps][kMaxE];
  __shared__ int ch[kThreads];
  __shared__ int sx[kThreads];  // the round's excess slot ids
  __shared__ int wpre[kWarps];
  __shared__ int s_total, s_chunk, s_first_bad, s_moved;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int64_t nslots = static_cast<int64_t>(S) * K;
  const int64_t ovf_row0 = static_cast<int64_t>(E) * C;
  const float kNegInf = __int_as_float(0xff800000);

  for (int e = tid; e < E; e += kThreads) {
    const int c = counts[e];
    room[e] = C - (c < C ? (c > 0 ? c : 0) : C);
  }
  for (int t = tid; t < S; t += kThreads) changed[t] = 0;
  if (tid == 0) {
    s_total = 0;
    s_moved = 0;
  }
  __syncthreads();

  // 1. the excess slots (overflow rows of the permutation), in slot order;
  //    each thread looks at kPer consecutive slots per pass
  constexpr int kPer = 8;
  for (int64_t base = 0; base < nslots; base += static_cast<int64_t>(kThreads) * kPer) {
    const int64_t s0 = base + static_cast<int64_t>(tid) * kPer;
    unsigned bits = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (s0 + j < nslots && row_of_slot[s0 + j] >= ovf_row0) bits |= 1u << j;
    const int n = __popc(bits);
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) wpre[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = wpre[lane];
      int winc = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, winc, off);
        if (lane >= off) winc += o;
      }
      wpre[lane] = winc - v;
      if (lane == 31) s_chunk = winc;
    }
    __syncthreads();
    int pos = s_total + wpre[warp] + incl - n;
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (bits & (1u << j)) ex[pos++] = static_cast<int32_t>(s0 + j);
    __syncthreads();
    if (tid == 0) s_total += s_chunk;
    __syncthreads();
  }
  const int n_ex = s_total;

  // 2. rounds over chunks of excess slots
  int base = 0;
  while (base < n_ex) {
    const int m = min(kThreads, n_ex - base);
    ch[tid] = -1;
    sx[tid] = tid < m ? ex[base + tid] : 0;
    for (int i = tid; i < kWarps * kMaxE; i += kThreads) (&wcnt[0][0])[i] = 0;
    if (tid == 0) s_first_bad = m;
    __syncthreads();
    {
      // groups of kG lanes; group g takes the chunk's slots from the first run
      // start at or after kSpan*g up to the first run start at or after
      // kSpan*(g+1), so a token's slots stay in one group and are picked in k
      // order.  Lane q of a group holds experts q, q + kG, q + 2 kG, ...
      auto run_start = [&](int i) {  // first i' >= i that starts a token's run (or m)
        while (i < m && i > 0 && sx[i - 1] / K == sx[i] / K) ++i;
        return i < m ? i : m;
      };
      const int g = tid / kG, q = tid % kG;
      const int i0 = g == 0 ? 0 : run_start(min(kSpan * g, m));
      const int i1 = run_start(min(kSpan * (g + 1), m));
      // the longest range of the warp's groups sets the warp's step count
      int steps = i1 - i0;
#pragma unroll
      for (int off = kG; off < 32; off <<= 1) steps = max(steps, __shfl_xor_sync(0xFFFFFFFFu, steps, off));
      uint32_t held = 0;  // bit r: expert q + kG*r is held by the current token
      int cur_t = -1;
      for (int step = 0; step < steps; ++step) {
        const int i = i0 + step;
        const bool act = i < i1;
        const int s = act ? sx[i] : 0;
        const int t = s / K;
        if (act && t != cur_t) {  // the token's current experts, loads issued in batches of 8
          cur_t = t;
          held = 0;
          const int32_t* row = topk_idx + static_cast<int64_t>(t) * K;
          for (int k0 = 0; k0 < K; k0 += 8) {
            int ev[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) ev[u] = k0 + u < K ? row[k0 + u] : -1;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              if (ev[u] >= 0 && ev[u] < E && ev[u] % kG == q) held |= 1u << (ev[u] / kG);
          }
        }
        // the best candidate with room that the token does not hold; key loads in batches of 8
        float bv = kNegInf;
        int be = 0x7fffffff;
        if (act) {
          const float* key = cand_key + static_cast<int64_t>(t) * E;
          for (int r0 = 0; r0 * kG < E; r0 += 8) {
            float kv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int e = (r0 + u) * kG + q;
              kv[u] = e < E ? __ldg(key + e) : kNegInf;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int r = r0 + u, e = r * kG + q;
              if (!(kv[u] > kNegInf) || ((held >> r) & 1u) || room[e] <= 0) continue;
              if (kv[u] > bv || (kv[u] == bv && e < be)) {
                bv = kv[u];
                be = e;
              }
            }
          }
        }
#pragma unroll
        for (int off = kG / 2; off >= 1; off >>= 1) {
          const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
          const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
          if (ov > bv || (ov == bv && oe < be)) {
            bv = ov;
            be = oe;
          }
        }
        if (act) {
          const int best = bv > kNegInf ? be : -1;
          if (q == 0) ch[i] = best;
          if (best >= 0 && best % kG == q) held |= 1u << (best / kG);
        }
      }
    }
    __syncthreads();
    // rank of each pick among the earlier picks of the same expert in this chunk
    const int c = tid < m ? ch[tid] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, c);
    const int wrank = __popc(peers & lt_mask);
    if (c >= 0 && wrank == 0) wcnt[warp][c] = __popc(peers);
    __syncthreads();
    bool bad = false;
    if (c >= 0) {
      int rank = wrank;
      for (int w = 0; w < warp; ++w) rank += wcnt[w][c];
      bad = rank >= room[c];
    }
    if (bad) atomicMin(&s_first_bad, tid);
    __syncthreads();
    const int p = s_first_bad;  // >= 1: the chunk's first pick always fits
    if (tid < p && c >= 0) {
      const int s = ex[base + tid];
      topk_idx[s] = c;
      atomicSub(&room[c], 1);
      changed[s / K] = 1;
      atomicAdd(&s_moved, 1);
    }
    __syncthreads();
    base += p;
  }
  if (tid == 0 && status != nullptr && s_moved > 0) atomicAdd(&status->counters[MOE_CNT_REROUTED], s_moved);
}

}  // namespace

cudaError_t launch_reroute_assign(int S, int E, int K, int capacity, int32_t* topk_idx, const float* cand_key,
                                  const int32_t* counts, const int32_t* row_of_slot, int32_t* ex_scratch,
                                  int32_t* changed, StatusBlock* status, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  if (E < 1 || E > kMaxE || K < 1 || K > 32 || capacity <= 0) return cudaErrorInvalidValue;
  reroute_assign_kernel<<<1, kThreads, 0, stream>>>(S, E, K, capacity, topk_idx, cand_key, counts, row_of_slot,
                                                    ex_scratch, changed, status);
  return cudaGetLastError();
}

}  // namespace moe
