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
// the room left at the start of the round (one thread per slot over the
// token's whole key row; the later slots of a token with several excess slots
// in the chunk are then fixed up in k order, each excluding the earlier
// picks), the picks are ranked per expert in slot order, and the longest
// prefix of slots whose pick still fits is committed.  A pick made against the round's room
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

// The best candidate expert of excess slot s with room left (room[e] > 0),
// a finite key, not held by the slot's token (its current K experts) and not
// in extra[0..n_extra): highest key, ties to the lower index; -1 if none.
// The key row is read with 16-byte loads issued before the comparisons.
__device__ int best_pick(int s, int E, int K, const int32_t* topk_idx, const float* cand_key, const int* room,
                         const int* extra, int n_extra) {
  const float kNegInf = __int_as_float(0xff800000);
  const int t = s / K;
  uint32_t held[kMaxE / 32];
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i) held[i] = 0;
  for (int k = 0; k < K; ++k) {
    const int e = topk_idx[static_cast<int64_t>(t) * K + k];
    if (e >= 0 && e < E) held[e >> 5] |= 1u << (e & 31);
  }
  for (int i = 0; i < n_extra; ++i) held[extra[i] >> 5] |= 1u << (extra[i] & 31);
  const float* row = cand_key + static_cast<int64_t>(t) * E;
  float bv = kNegInf;
  int be = -1;
  // E is a multiple of 4 here (whole 16-byte loads) or handled one by one
  const int e4 = (E % 4 == 0) ? E : 0;
  for (int e0 = 0; e0 < e4; e0 += 32) {
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      v[j] = (e0 + 4 * j < e4) ? __ldg(reinterpret_cast<const float4*>(row + e0 + 4 * j))
                               : make_float4(kNegInf, kNegInf, kNegInf, kNegInf);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float kv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int e = e0 + 4 * j + c;
        if (e >= E || !(kv[c] > kNegInf) || ((held[e >> 5] >> (e & 31)) & 1u) || room[e] <= 0) continue;
        if (kv[c] > bv) {  // ascending e: a tie keeps the lower index
          bv = kv[c];
          be = e;
        }
      }
    }
  }
  for (int e = e4; e < E; ++e) {
    const float kv = __ldg(row + e);
    if (!(kv > kNegInf) || ((held[e >> 5] >> (e & 31)) & 1u) || room[e] <= 0) continue;
    if (kv > bv) {
      bv = kv;
      be = e;
    }
  }
  return be;
}

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
      // one thread per slot: the best candidate with room that the token does
      // not hold, over the token's whole key row (16-byte loads, all issued
      // together); then the slots of a token that has several excess slots
      // in this chunk are fixed up in k order, each excluding the earlier
      // ones' picks
      if (tid < m) ch[tid] = best_pick(sx[tid], E, K, topk_idx, cand_key, room, nullptr, 0);
      __syncthreads();
      if (tid < m && (tid == 0 || sx[tid - 1] / K != sx[tid] / K) && tid + 1 < m && sx[tid + 1] / K == sx[tid] / K) {
        int taken[32];
        int nt = 0;
        if (ch[tid] >= 0) taken[nt++] = ch[tid];
        for (int j = tid + 1; j < m && sx[j] / K == sx[tid] / K; ++j) {
          bool clash = false;
          for (int i = 0; i < nt; ++i) clash |= ch[j] == taken[i];
          if (clash) ch[j] = best_pick(sx[j], E, K, topk_idx, cand_key, room, taken, nt);
          if (ch[j] >= 0 && nt < 32) taken[nt++] = ch[j];
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
