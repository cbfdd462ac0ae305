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
// The visit order makes this a serial assignment, but its picks only change
// when an expert runs out of room, and that happens at most once per expert.
// So it runs in epochs:
//  1. every excess slot picks against the room at the start (all SMs, one
//     thread per token taking its excess slots in k order, each excluding the
//     token's experts and its earlier picks), and the excess slots are listed;
//  2. one CTA then repeats: find the first slot whose pick overflows its
//     expert's room (per-expert counts of the uncommitted picks by token
//     segment, then by sub-range of that segment, then a scan of one
//     sub-range); commit every pick before it (these are the serial picks: no
//     expert they chose was full when they were made) by moving counts only;
//     the experts left without room drop out, and only the uncommitted slots
//     that picked one of them pick again (with the later slots of their token
//     that now clash).  Every epoch but the last fills at least one expert,
//     so there are at most E + 1;
//  3. the final picks become the slots' experts (all SMs).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kMaxE = 256;
constexpr int kMaskWords = kMaxE / 32;
constexpr int kPickThreads = 256;
constexpr int kThreads = 512;
constexpr int kSegs = kThreads / 32;  // token segments, one per warp of the commit CTA
constexpr int kScanSlots = 512;       // slots the scanning warp loads at once
constexpr size_t kCommitSmemMax = 227 * 1024;  // shared memory of the commit CTA (picks included)
constexpr int kNone = -1;             // excess slot without a candidate
constexpr int kKept = -2;             // slot within its expert's capacity

__device__ __forceinline__ bool bit_of(const uint32_t* m, int e) { return (m[e >> 5] >> (e & 31)) & 1u; }

// Word i of a per-thread expert mask, and setting bit e of it, by unrolled
// selects, so the mask stays in registers whatever i or e are.
__device__ __forceinline__ uint32_t word_of(const uint32_t (&m)[kMaskWords], int i) {
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < kMaskWords; ++j) r = (i == j) ? m[j] : r;
  return r;
}
__device__ __forceinline__ void set_bit(uint32_t (&m)[kMaskWords], int e) {
#pragma unroll
  for (int j = 0; j < kMaskWords; ++j)
    if ((e >> 5) == j) m[j] |= 1u << (e & 31);
}
__device__ __forceinline__ bool has_bit(const uint32_t (&m)[kMaskWords], int e) {
  return (word_of(m, e >> 5) >> (e & 31)) & 1u;
}

// The best candidate of token t: highest key among experts in `avail`, not in
// `held`, with a key above -inf; ties to the lower index; kNone if none.  The
// key row is read 64 experts at a time with sixteen 16-byte loads in flight.
__device__ int best_candidate(const float* __restrict__ row, int E, const uint32_t* avail,
                              const uint32_t (&held)[kMaskWords]) {
  const float kNegInf = __int_as_float(0xff800000);
  float bv = kNegInf;
  int be = kNone;
  const int e4 = (E % 4 == 0) ? E : 0;
  for (int e0 = 0; e0 < e4; e0 += 64) {
    float4 v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = (e0 + 4 * j < e4) ? __ldg(reinterpret_cast<const float4*>(row + e0 + 4 * j))
                               : make_float4(kNegInf, kNegInf, kNegInf, kNegInf);
    const int w = e0 >> 5;
    const uint64_t av = static_cast<uint64_t>(avail[w]) | (e0 + 32 < E ? static_cast<uint64_t>(avail[w + 1]) << 32 : 0);
    const uint64_t hb = static_cast<uint64_t>(word_of(held, w)) | (static_cast<uint64_t>(word_of(held, w + 1)) << 32);
    const uint64_t ok = av & ~hb;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float kv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int e = e0 + 4 * j + c;
        if (e >= E || !(kv[c] > bv) || !((ok >> (4 * j + c)) & 1u)) continue;
        bv = kv[c];  // strictly greater in ascending e: a tie keeps the lower index
        be = e;
      }
    }
  }
  for (int e = e4; e < E; ++e) {
    const float kv = __ldg(row + e);
    if (!(kv > bv) || has_bit(held, e) || !bit_of(avail, e)) continue;
    bv = kv;
    be = e;
  }
  return be;
}

// Bit e set for every expert the token's K slots hold (vec: 16-byte loads,
// K a multiple of 4 and the row 16-byte aligned).
__device__ __forceinline__ void held_of(const int32_t* __restrict__ idx_row, int K, int E, bool vec,
                                        uint32_t (&held)[kMaskWords]) {
#pragma unroll
  for (int i = 0; i < kMaskWords; ++i) held[i] = 0;
  auto add = [&](int e) {
    if (e >= 0 && e < E) set_bit(held, e);
  };
  if (vec) {
    int4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (4 * j < K) v[j] = reinterpret_cast<const int4*>(idx_row)[j];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (4 * j < K) {
        add(v[j].x); add(v[j].y); add(v[j].z); add(v[j].w);
      }
  } else {
    for (int k = 0; k < K; ++k) add(idx_row[k]);
  }
}

// Bit k set for every slot of the token in the overflow region (row >=
// ovf_row0); vec as for held_of.
__device__ __forceinline__ uint32_t excess_mask(const int32_t* __restrict__ ros_row, int K, int64_t ovf_row0,
                                                bool vec) {
  uint32_t m = 0;
  if (vec) {
    int4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (4 * j < K) v[j] = reinterpret_cast<const int4*>(ros_row)[j];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (4 * j < K) {
        m |= (v[j].x >= ovf_row0 ? 1u : 0u) << (4 * j);
        m |= (v[j].y >= ovf_row0 ? 1u : 0u) << (4 * j + 1);
        m |= (v[j].z >= ovf_row0 ? 1u : 0u) << (4 * j + 2);
        m |= (v[j].w >= ovf_row0 ? 1u : 0u) << (4 * j + 3);
      }
  } else {
    for (int k = 0; k < K; ++k) m |= (ros_row[k] >= ovf_row0 ? 1u : 0u) << k;
  }
  return m;
}

// Calls f(s, pick[s]) for every slot s in [lo, hi), reading the pick buffer
// in 16-byte pieces (four slots; the buffer is 16-byte aligned), four pieces
// in flight per thread: thread `idx` of `nthreads` takes pieces idx,
// idx + nthreads, ...
template <typename F>
__device__ __forceinline__ void for_picks(const int32_t* __restrict__ pick, int64_t lo, int64_t hi, int idx,
                                          int nthreads, F&& f) {
  constexpr int U = 4;
  if (lo >= hi) return;
  const int64_t q0 = lo >> 2, q1 = (hi + 3) >> 2;
  const int4* p4 = reinterpret_cast<const int4*>(pick);
  for (int64_t qb = q0 + idx; qb < q1; qb += U * static_cast<int64_t>(nthreads)) {
    int4 v[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t q = qb + j * static_cast<int64_t>(nthreads);
      v[j] = q < q1 ? p4[q] : make_int4(kKept, kKept, kKept, kKept);
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t s0 = (qb + j * static_cast<int64_t>(nthreads)) * 4;
      const int pv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (s0 + c >= lo && s0 + c < hi) f(s0 + c, pv[c]);
    }
  }
}


// best_candidate over a key row already in registers (E <= 64, E a multiple
// of 4): the same choice without reading memory.
__device__ __forceinline__ int best_candidate_regs(const float4 (&v)[16], int E, const uint32_t* avail,
                                                   const uint32_t (&held)[kMaskWords]) {
  const float kNegInf = __int_as_float(0xff800000);
  float bv = kNegInf;
  int be = kNone;
  const uint64_t av = static_cast<uint64_t>(avail[0]) | (E > 32 ? static_cast<uint64_t>(avail[1]) << 32 : 0);
  const uint64_t ok = av & ~(static_cast<uint64_t>(held[0]) | (static_cast<uint64_t>(held[1]) << 32));
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float kv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = 4 * j + c;
      if (e >= E || !(kv[c] > bv) || !((ok >> e) & 1u)) continue;
      bv = kv[c];
      be = e;
    }
  }
  return be;
}

// Calls f(s, pick[s]) for every entry s of the excess-slot list ex[0, n)
// (16-byte aligned): thread `idx` of `nthreads` takes entries in pieces of
// four, four pieces in flight, then the four picks of each piece.
template <typename F>
__device__ __forceinline__ void for_excess(const int32_t* __restrict__ ex, int n, const int32_t* __restrict__ pick,
                                           int idx, int nthreads, F&& f) {
  constexpr int U = 4;
  const int q1 = (n + 3) >> 2;
  const int4* e4 = reinterpret_cast<const int4*>(ex);
  for (int qb = idx; qb < q1; qb += U * nthreads) {
    int4 v[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int q = qb + j * nthreads;
      v[j] = q < q1 ? e4[q] : make_int4(-1, -1, -1, -1);
    }
    int sv[4 * U], pv[4 * U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int base = 4 * (qb + j * nthreads);
      sv[4 * j] = base < n ? v[j].x : -1;
      sv[4 * j + 1] = base + 1 < n ? v[j].y : -1;
      sv[4 * j + 2] = base + 2 < n ? v[j].z : -1;
      sv[4 * j + 3] = base + 3 < n ? v[j].w : -1;
    }
#pragma unroll
    for (int i = 0; i < 4 * U; ++i) pv[i] = sv[i] >= 0 ? pick[sv[i]] : kKept;
#pragma unroll
    for (int i = 0; i < 4 * U; ++i)
      if (sv[i] >= 0) f(static_cast<int64_t>(sv[i]), pv[i]);
  }
}

// Where the commit kernel keeps the picks: in shared memory as one signed
// byte per slot (E <= 127 and every slot fitting), kept in step with the
// global int32 copy the apply kernel reads; or in the global copy alone.
template <bool SM>
struct Picks;

template <>
struct Picks<true> {
  int8_t* s;   // shared, 16-byte aligned
  int32_t* g;  // global copy
  __device__ int get(int64_t i) const { return s[i]; }
  __device__ void set(int64_t i, int v) const {
    s[i] = static_cast<int8_t>(v);
    g[i] = v;
  }
  // f(slot, pick) for every slot in [lo, hi); thread idx of nthreads takes
  // 16-slot pieces idx, idx + nthreads, ...
  template <typename F>
  __device__ void for_range(int64_t lo, int64_t hi, int idx, int nthreads, F&& f) const {
    if (lo >= hi) return;
    const uint4* s4 = reinterpret_cast<const uint4*>(s);
    for (int64_t q = (lo >> 4) + idx; q < ((hi + 15) >> 4); q += nthreads) {
      const uint4 v = s4[q];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int64_t slot = q * 16 + c;
        if (slot >= lo && slot < hi) f(slot, static_cast<int>(static_cast<int8_t>(w[c >> 2] >> (8 * (c & 3)))));
      }
    }
  }
};

template <>
struct Picks<false> {
  int32_t* g;
  __device__ int get(int64_t i) const { return g[i]; }
  __device__ void set(int64_t i, int v) const { g[i] = v; }
  template <typename F>
  __device__ void for_range(int64_t lo, int64_t hi, int idx, int nthreads, F&& f) const {
    for_picks(g, lo, hi, idx, nthreads, f);
  }
};

// Step 1: the picks of every excess slot against the starting room, and the
// list of the excess slots (any order; ex_count counts them).  pick[s] =
// expert, kNone, or kKept for slots within capacity.  Warps walk 32
// consecutive tokens at a time, so one lane per warp reserves the list
// entries of all 32.
__global__ void __launch_bounds__(kPickThreads)
    reroute_pick_kernel(int S, int E, int K, int C, const int32_t* __restrict__ topk_idx,
                        const float* __restrict__ cand_key, const int32_t* __restrict__ counts,
                        const int32_t* __restrict__ row_of_slot, int32_t* __restrict__ pick,
                        int32_t* __restrict__ changed, int32_t* __restrict__ claim, int32_t* __restrict__ ex,
                        int32_t* __restrict__ ex_count, int8_t* __restrict__ pick8, bool vec) {
  __shared__ uint32_t avail[kMaskWords];
  if (threadIdx.x < kMaskWords) avail[threadIdx.x] = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (counts[e] < C) atomicOr(&avail[e >> 5], 1u << (e & 31));
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t ovf_row0 = static_cast<int64_t>(E) * C;
  const int stride = gridDim.x * blockDim.x;
  for (int tb = blockIdx.x * blockDim.x + (threadIdx.x & ~31); tb < S; tb += stride) {
    const int t = tb + lane;
    const bool live = t < S;
    const int64_t s0 = static_cast<int64_t>(t) * K;
    uint32_t exm = 0;
    if (live) {
      changed[t] = 0;
      claim[t] = 0;
      exm = excess_mask(row_of_slot + s0, K, ovf_row0, vec);
    }
    // list positions: one atomic per warp
    const int n = __popc(exm);
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += o;
    }
    int base = 0;
    if (lane == 31 && incl > 0) base = atomicAdd(ex_count, incl);
    base = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - n;
    if (!live) continue;
    if (exm == 0) {
      for (int k = 0; k < K; ++k) {
        pick[s0 + k] = kKept;
        if (pick8 != nullptr) pick8[s0 + k] = static_cast<int8_t>(kKept);
      }
      continue;
    }
    uint32_t held[kMaskWords];
    held_of(topk_idx + s0, K, E, vec, held);
    for (int k = 0; k < K; ++k) {
      int p = kKept;
      if ((exm >> k) & 1u) {
        p = best_candidate(cand_key + static_cast<int64_t>(t) * E, E, avail, held);
        if (p >= 0) set_bit(held, p);
        ex[base++] = static_cast<int32_t>(s0 + k);
      }
      pick[s0 + k] = p;
      if (pick8 != nullptr) pick8[s0 + k] = static_cast<int8_t>(p);
    }
  }
}

// Final step: the picks become the slots' experts; changed[t] marks the
// tokens with a moved slot, and the moved slots are counted.
__global__ void __launch_bounds__(kPickThreads)
    reroute_apply_kernel(int K, const int32_t* __restrict__ ex, const int32_t* __restrict__ ex_count,
                         const int32_t* __restrict__ pick, int32_t* __restrict__ topk_idx,
                         int32_t* __restrict__ changed, StatusBlock* status) {
  const int n = *ex_count;
  int moved = 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int s = ex[i];
    const int p = pick[s];
    if (p >= 0) {
      topk_idx[s] = p;
      changed[s / K] = 1;
      ++moved;
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) moved += __shfl_xor_sync(0xFFFFFFFFu, moved, off);
  if ((threadIdx.x & 31) == 0 && moved > 0 && status != nullptr) atomicAdd(&status->counters[MOE_CNT_REROUTED], moved);
}

// Step 2: the epochs, on one CTA.  A pick counts as committed once every
// earlier overflow has been resolved; commits only move counts (room and the
// segment counts), and the apply kernel writes the final experts at the end.
struct CommitSmem {
  int cnt[kSegs][kMaxE];  // uncommitted picks of each expert in each token segment
  int sub[kSegs][kMaxE];  // the same within the kSegs sub-ranges of one segment
  int room[kMaxE];
  int seg_e[kMaxE];       // segment holding expert e's first overflowing pick (kSegs: none)
  int need_e[kMaxE];      // e's uncommitted picks there before it
  int sub_e[kMaxE];       // sub-range of that pick, and the picks before it there
  int need2_e[kMaxE];
  int run[kMaxE];         // picks of each expert in the scanned sub-range before the overflow
  uint32_t avail[kMaskWords];
  uint32_t full[kMaskWords];  // experts that ran out of room in this epoch
  int min_seg, min_sub;
  long long first_bad;
  int nlist;     // tokens listed for re-picking in this epoch
  int nf;        // experts that ran out of room in this epoch, and the first four of them
  int flist[4];
};

// The excess slots of token t from slot `first` on pick again, in k order: a
// slot whose pick ran out of room (in `full`), or that now clashes with an
// earlier slot's new pick, takes the best candidate among the experts still
// available; the token's experts and all its earlier picks are held.  The
// segment counts follow every change.  With E <= 64 the key row is read once
// into registers.
template <bool SM>
__device__ __forceinline__ void repick_token(int t, int64_t first, int E, int K, bool vec, int seg,
                                             const int32_t* __restrict__ topk_idx,
                                             const float* __restrict__ cand_key, const Picks<SM>& pick,
                                             CommitSmem& sm) {
  const int64_t s0 = static_cast<int64_t>(t) * K;
  const int k0 = static_cast<int>((first > s0 ? first : s0) - s0);
  const float* row = cand_key + static_cast<int64_t>(t) * E;
  const bool regs = E <= 64 && E % 4 == 0;
  const float kNegInf = __int_as_float(0xff800000);
  float4 kv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j)
    kv[j] = (regs && 4 * j < E) ? __ldg(reinterpret_cast<const float4*>(row) + j)
                                : make_float4(kNegInf, kNegInf, kNegInf, kNegInf);
  uint32_t held[kMaskWords];
  held_of(topk_idx + s0, K, E, vec, held);
  // the picks are read slot by slot: an array of them indexed by k would live
  // in local memory, which with the picks filling shared memory misses L1
  for (int k = 0; k < K; ++k) {
    int p = pick.get(s0 + k);
    if (p == kKept) continue;
    if (k >= k0 && p >= 0 && (bit_of(sm.full, p) || has_bit(held, p))) {
      const int q = regs ? best_candidate_regs(kv, E, sm.avail, held) : best_candidate(row, E, sm.avail, held);
      atomicSub(&sm.cnt[seg][p], 1);
      if (q >= 0) atomicAdd(&sm.cnt[seg][q], 1);
      pick.set(s0 + k, q);
      p = q;
    }
    if (p >= 0) set_bit(held, p);
  }
}

template <bool SM>
__global__ void __launch_bounds__(kThreads, 1)
    reroute_commit_kernel(int S, int E, int K, int C, const int32_t* __restrict__ topk_idx,
                          const float* __restrict__ cand_key, const int32_t* __restrict__ counts,
                          int32_t* __restrict__ pick_g, const int8_t* __restrict__ pick8,
                          const int32_t* __restrict__ ex, const int32_t* __restrict__ ex_count,
                          int32_t* __restrict__ claim, int32_t* __restrict__ list, bool vec, StatusBlock* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  CommitSmem& sm = *reinterpret_cast<CommitSmem*>(smem_raw);
  Picks<SM> pick;
  if constexpr (SM) {
    pick.s = reinterpret_cast<int8_t*>(smem_raw + ((sizeof(CommitSmem) + 15) & ~size_t(15)));
    pick.g = pick_g;
  } else {
    pick.g = pick_g;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nslots = static_cast<int64_t>(S) * K;
  const int n_ex = *ex_count;
  const int seg_len = (S + kSegs - 1) / kSegs;  // tokens per segment
  auto seg_of = [&](int64_t s) { return static_cast<int>((s / K) / seg_len); };
  auto seg_begin = [&](int w) { return static_cast<int64_t>(min(S, w * seg_len)) * K; };

  for (int i = tid; i < kSegs * kMaxE; i += kThreads) (&sm.cnt[0][0])[i] = 0;
  if (tid < kMaskWords) sm.avail[tid] = 0;
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) {
    const int c = counts[e];
    sm.room[e] = C - (c < C ? (c > 0 ? c : 0) : C);
    if (sm.room[e] > 0) atomicOr(&sm.avail[e >> 5], 1u << (e & 31));
  }
  if constexpr (SM) {
    // the byte copy of the picks into shared memory
    const int64_t n16 = (nslots + 15) >> 4;
    for (int64_t i = tid; i < n16; i += kThreads)
      reinterpret_cast<uint4*>(pick.s)[i] = reinterpret_cast<const uint4*>(pick8)[i];
    __syncthreads();
    pick.for_range(0, nslots, tid, kThreads, [&](int64_t s, int p) {
      if (p >= 0) atomicAdd(&sm.cnt[seg_of(s)][p], 1);
    });
  } else {
    // the picks of each segment, from the excess-slot list
    for_excess(ex, n_ex, pick_g, tid, kThreads, [&](int64_t s, int p) {
      if (p >= 0) atomicAdd(&sm.cnt[seg_of(s)][p], 1);
    });
  }
  __syncthreads();

  int64_t start = 0;  // first uncommitted slot
  bool ok = true;
  for (int epoch = 0; epoch <= E + 1; ++epoch) {
    // 1. for each available expert, the segment of its first overflowing pick
    if (tid == 0) {
      sm.min_seg = kSegs;
      sm.min_sub = kSegs;
      sm.first_bad = nslots;
      sm.nlist = 0;
      sm.nf = 0;
    }
    for (int e = tid; e < E; e += kThreads) {
      int seg = kSegs, acc = 0, need = 0;
      if (bit_of(sm.avail, e)) {
        for (int w = 0; w < kSegs; ++w) {
          const int c = sm.cnt[w][e];
          if (acc + c > sm.room[e]) {
            seg = w;
            need = sm.room[e] - acc;
            break;
          }
          acc += c;
        }
      }
      sm.seg_e[e] = seg;
      sm.need_e[e] = need;
      sm.run[e] = 0;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads)
      if (sm.seg_e[e] < kSegs) atomicMin(&sm.min_seg, sm.seg_e[e]);
    for (int i = tid; i < kSegs * kMaxE; i += kThreads) (&sm.sub[0][0])[i] = 0;
    __syncthreads();
    const int ms = sm.min_seg;
    if (ms >= kSegs) break;  // no pick overflows: every remaining pick stands
    // 2. the exact slot: sub-range counts of all picks within segment ms, then
    //    a scan of the sub-range holding the first overflow, in slot order
    const int64_t a = max(seg_begin(ms), start), b = seg_begin(ms + 1);
    const int64_t span = (b - a + kSegs - 1) / kSegs;
    {
      const int64_t lo = min(b, a + warp * span), hi = min(b, lo + span);
      pick.for_range(lo, hi, lane, 32, [&](int64_t, int p) {
        if (p >= 0) atomicAdd(&sm.sub[warp][p], 1);
      });
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
      int w_hit = kSegs, acc = 0, need2 = 0;
      if (sm.seg_e[e] == ms) {
        for (int w = 0; w < kSegs; ++w) {
          const int c = sm.sub[w][e];
          if (acc + c > sm.need_e[e]) {
            w_hit = w;
            need2 = sm.need_e[e] - acc;
            break;
          }
          acc += c;
        }
        atomicMin(&sm.min_sub, w_hit);
      }
      sm.sub_e[e] = w_hit;
      sm.need2_e[e] = need2;
    }
    __syncthreads();
    const int wm = sm.min_sub;
    if (warp == wm) {
      // loaded kScanSlots slots at a time (all loads in flight together),
      // each piece scanned 32 slots at a time in slot order; run[] counts the
      // picks of every expert before the overflowing one
      const int64_t slo = min(b, a + wm * span), shi = min(b, slo + span);
      const unsigned lt = (1u << lane) - 1u;
      bool found = false;
      for (int64_t c0 = slo; c0 < shi && !found; c0 += kScanSlots) {
        int pv[kScanSlots / 32];
#pragma unroll
        for (int j = 0; j < kScanSlots / 32; ++j) {
          const int64_t s = c0 + 32 * j + lane;
          pv[j] = s < shi ? pick.get(s) : kKept;
        }
#pragma unroll
        for (int j = 0; j < kScanSlots / 32; ++j) {
          const int p = pv[j];
          const bool cand = p >= 0 && sm.seg_e[p] == ms && sm.sub_e[p] == wm;
          const unsigned peers = __match_any_sync(0xFFFFFFFFu, p);
          const int rank = __popc(peers & lt);
          const bool hit = cand && sm.run[p] + rank == sm.need2_e[p];
          const unsigned hits = __ballot_sync(0xFFFFFFFFu, hit);
          // picks before the first hit (all of them when there is none)
          const unsigned before = hits != 0 ? (1u << (__ffs(hits) - 1)) - 1u : 0xFFFFFFFFu;
          const unsigned pb = peers & before;
          if (p >= 0 && ((before >> lane) & 1u) && (pb & lt) == 0) sm.run[p] += __popc(pb);
          if (hits != 0) {
            if (lane == 0) sm.first_bad = c0 + 32 * j + __ffs(hits) - 1;
            found = true;
            break;
          }
          __syncwarp();
        }
      }
    }
    __syncthreads();
    const int64_t P = sm.first_bad;
    if (P >= nslots) {  // the counts promised an overflow in this segment: cannot happen
      ok = false;
      break;
    }
    // 3. commit the picks of [start, P): counts only
    for (int e = tid; e < E; e += kThreads) {
      int c = 0;
      for (int w = 0; w < ms; ++w) {
        c += sm.cnt[w][e];
        sm.cnt[w][e] = 0;
      }
      int cm = sm.run[e];
      for (int w = 0; w < wm; ++w) cm += sm.sub[w][e];
      sm.cnt[ms][e] -= cm;
      sm.room[e] -= c + cm;
    }
    if (tid < kMaskWords) sm.full[tid] = 0;
    __syncthreads();
    start = P;
    // 4. experts left without room drop out
    for (int e = tid; e < E; e += kThreads)
      if (bit_of(sm.avail, e) && sm.room[e] <= 0) {
        atomicOr(&sm.full[e >> 5], 1u << (e & 31));
        const int i = atomicAdd(&sm.nf, 1);
        if (i < 4) sm.flist[i] = e;
      }
    __syncthreads();
    if (tid < kMaskWords) sm.avail[tid] &= ~sm.full[tid];
    __syncthreads();
    // 5. the tokens with an uncommitted slot that picked a full expert pick
    //    again: the first thread to see such a slot claims the token for this
    //    epoch and lists it; then the listed tokens are re-picked, one per
    //    thread (so the threads of a warp re-pick side by side)
    auto claim_slot = [&](int64_t s, int p) {
      if (s < P || p < 0 || !bit_of(sm.full, p)) return;
      const int t = static_cast<int>(s / K);
      if (atomicMax(&claim[t], epoch + 1) < epoch + 1) list[atomicAdd(&sm.nlist, 1)] = t;
    };
    if constexpr (SM) {
      if (sm.nf <= 4 && 16 % K == 0) {
        // a 16-slot piece holds whole tokens, so one thread sees all of a
        // token's slots and lists it without a claim; four picks per word are
        // compared at once with the (at most four) experts that filled up
        uint32_t fb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) fb[i] = 0x01010101u * static_cast<uint32_t>(sm.flist[i < sm.nf ? i : 0]);
        const uint4* s4 = reinterpret_cast<const uint4*>(pick.s);
        const uint32_t tmask = (K >= 16) ? 0xFFFFu : ((1u << K) - 1u);
        for (int64_t q = (P >> 4) + tid; q < ((nslots + 15) >> 4); q += kThreads) {
          const uint4 v = s4[q];
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          uint32_t hit = 0;  // bit c: slot q*16 + c picked a full expert
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t m = 0;
#pragma unroll
            for (int f = 0; f < 4; ++f) m |= __vcmpeq4(wv[i], fb[f]);
            hit |= ((m & 1u) | ((m >> 7) & 2u) | ((m >> 14) & 4u) | ((m >> 21) & 8u)) << (4 * i);
          }
          if (hit == 0) continue;
          const int64_t s_lo = q * 16;
          if (s_lo < P) hit &= ~((1u << static_cast<int>(P - s_lo)) - 1u);  // committed slots
          if (s_lo + 16 > nslots) hit &= (1u << static_cast<int>(nslots - s_lo)) - 1u;
          for (int c0 = 0; c0 < 16; c0 += K)
            if ((hit >> c0) & tmask) list[atomicAdd(&sm.nlist, 1)] = static_cast<int>((s_lo + c0) / K);
        }
      } else {
        pick.for_range(P, nslots, tid, kThreads, claim_slot);
      }
    } else {
      for_excess(ex, n_ex, pick_g, tid, kThreads, claim_slot);
    }
    __syncthreads();
    const int nl = sm.nlist;
    for (int i = tid; i < nl; i += kThreads) {
      const int t = list[i];
      repick_token<SM>(t, P, E, K, vec, seg_of(static_cast<int64_t>(t) * K), topk_idx, cand_key, pick, sm);
    }
    __syncthreads();
  }
  if (!ok || sm.min_seg < kSegs) report(status, MOE_STATUS_DEBUG_CHECK, -1);
}

}  // namespace

cudaError_t launch_reroute_assign(int S, int E, int K, int capacity, int32_t* topk_idx, const float* cand_key,
                                  const int32_t* counts, const int32_t* row_of_slot, const RerouteScratch& w,
                                  int32_t* changed, StatusBlock* status, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  if (E < 1 || E > kMaxE || K < 1 || K > 32 || capacity <= 0) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(w.pick) & 15) != 0 || (reinterpret_cast<uintptr_t>(w.ex) & 15) != 0)
    return cudaErrorInvalidValue;
  const bool vec = K % 4 == 0 && (reinterpret_cast<uintptr_t>(topk_idx) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(row_of_slot) & 15) == 0;
  cudaError_t err = cudaMemsetAsync(w.ex_count, 0, sizeof(int32_t), stream);
  if (err != cudaSuccess) return err;
  const int want = (S + kPickThreads - 1) / kPickThreads;
  const int grid = want < 148 * 8 ? want : 148 * 8;
  reroute_pick_kernel<<<grid, kPickThreads, 0, stream>>>(S, E, K, capacity, topk_idx, cand_key, counts, row_of_slot,
                                                         w.pick, changed, w.claim, w.ex, w.ex_count,
                                                         E <= 127 ? w.pick8 : nullptr, vec);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  // the picks in shared memory when they fit (one byte each, E <= 127)
  const int64_t nslots = static_cast<int64_t>(S) * K;
  const size_t base = (sizeof(CommitSmem) + 15) & ~size_t(15);
  const size_t smem_sm = base + static_cast<size_t>((nslots + 15) & ~int64_t(15));
  const bool in_smem = E <= 127 && w.pick8 != nullptr && smem_sm <= kCommitSmemMax;
  const size_t smem = in_smem ? smem_sm : sizeof(CommitSmem);
  auto kern = in_smem ? reroute_commit_kernel<true> : reroute_commit_kernel<false>;
  if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) !=
      cudaSuccess)
    return err;
  kern<<<1, kThreads, smem, stream>>>(S, E, K, capacity, topk_idx, cand_key, counts, w.pick, w.pick8, w.ex,
                                      w.ex_count, w.claim, w.list, vec, status);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  reroute_apply_kernel<<<grid, kPickThreads, 0, stream>>>(K, w.ex, w.ex_count, w.pick, topk_idx, changed, status);
  return cudaGetLastError();
}

}  // namespace moe
