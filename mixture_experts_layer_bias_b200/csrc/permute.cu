// Grouping by expert: histogram -> prefix scan -> stable permutation, and the
// gather of token rows into expert-contiguous rows.
//
// jsqmd.com "第11章 MoE模型推理" 11.1.2 (the S*K expert forwards are grouped
// and merged by expert) and 11.2.1 (regroup the sequence into one
// sub-sequence per expert, restore the original order afterwards);
// ybb.press "MoE 推理工程深层实战" 2.2 (rows above a capacity go to an overflow
// buffer that is processed later; none is dropped).
//
// Four kernels, no atomics on row positions, so the permutation is
// deterministic and stable (rows of an expert follow slot order t*K + k):
//  1. count:   each CTA owns a chunk of whole tokens and writes its expert
//              histogram (shared-memory atomics; counts are order-free);
//  2. scan:    one CTA turns the chunk histograms into per-chunk bases
//              (exclusive prefix over chunks) and the expert offsets
//              (exclusive prefix over experts), plus the overflow split;
//  3. scatter: each CTA ranks its slots inside the chunk (warp match/popc,
//              then a prefix over warps) and writes row_of_slot / token_of_row;
//  4. gather:  one warp per token copies its row once from HBM to its K rows
//              with 16-byte vectors.
// Small batches (S*K <= 4096 slots) run steps 1-3 and the group tables of the
// GEMMs in one single-CTA kernel, and the gather with one CTA per token.
#include "common.cuh"
#include "kernels.h"
#include "pdl.cuh"
#include "route_select.cuh"

namespace moe {

namespace {

constexpr int kChunkSlots = 1024;  // slots per CTA (whole tokens)
constexpr int kSmallWarps = 32;
constexpr int kSmallSlots = 4096;  // the single-CTA permutation handles S*K up to this
constexpr int64_t kFoldGatherBytes = 256 << 10;  // ... and also copies the rows up to this many bytes
constexpr int kPermWarps = 8;
constexpr unsigned kFull = 0xFFFFFFFFu;

__global__ void __launch_bounds__(256)
    count_kernel(int S, int E, int K, int tok_per_chunk, const int32_t* __restrict__ topk_idx,
                 int32_t* __restrict__ chunk_hist, StatusBlock* status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * tok_per_chunk * K;
  const int64_t s1 = min(static_cast<int64_t>(S) * K, s0 + static_cast<int64_t>(tok_per_chunk) * K);
  int bad = 0;
  for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int e = topk_idx[s];
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      ++bad;
  }
  if (bad) report(status, MOE_STATUS_BAD_EXPERT_ID, MOE_CNT_BAD_ID, bad);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// Inclusive warp scan helper over one value per lane.
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = lane_id();
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(kFull, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Exclusive prefix of src[0..n) into dst[0..n], dst[n] = total, by warp 0.
__device__ void warp0_exclusive_scan(const int32_t* src, int32_t* dst, int n) {
  if (threadIdx.x >= 32) return;
  const int lane = lane_id();
  int carry = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int v = i < n ? src[i] : 0;
    const int incl = warp_incl_scan(v);
    if (i < n) dst[i] = carry + incl - v;
    carry += __shfl_sync(kFull, incl, 31);
  }
  if (lane == 0) dst[n] = carry;
}

// The chunk histograms of one expert are split into P = blockDim / E
// contiguous segments, one thread each: segment sums, a prefix over the
// segments, then a second pass writes the running (exclusive) chunk bases.
__global__ void __launch_bounds__(1024)
    scan_kernel(int E, int num_chunks, int capacity, int32_t* __restrict__ chunk_hist, int32_t* __restrict__ counts,
                int32_t* __restrict__ offsets, StatusBlock* status) {
  extern __shared__ int32_t sm[];
  const int P = blockDim.x / E;        // >= 1 since E <= 256 < blockDim
  int32_t* part = sm;                  // [P][E] segment sums
  int32_t* cnt = sm + P * E;           // [E]
  int32_t* ovf = cnt + E;              // [E]
  int32_t* tmp = ovf + E;              // [E+1]
  const int tid = threadIdx.x;
  const int e = tid % E, pi = tid / E;
  const bool active = pi < P;
  const int seg = (num_chunks + P - 1) / P;
  const int c0 = min(num_chunks, pi * seg), c1 = min(num_chunks, c0 + seg);
  int local = 0;
  if (active)
    for (int c = c0; c < c1; ++c) local += chunk_hist[static_cast<int64_t>(c) * E + e];
  if (active) part[pi * E + e] = local;
  __syncthreads();
  if (active) {
    int run = 0;
    for (int q = 0; q < pi; ++q) run += part[q * E + e];
    for (int c = c0; c < c1; ++c) {
      const int64_t i = static_cast<int64_t>(c) * E + e;
      const int v = chunk_hist[i];
      chunk_hist[i] = run;
      run += v;
    }
    if (pi == P - 1) {
      cnt[e] = run;
      counts[e] = run;
      ovf[e] = capacity > 0 ? max(run - capacity, 0) : 0;
    }
  }
  __syncthreads();
  warp0_exclusive_scan(cnt, tmp, E);
  __syncthreads();
  for (int i = tid; i <= E; i += blockDim.x) offsets[i] = tmp[i];
  if (capacity > 0) {
    __syncthreads();
    warp0_exclusive_scan(ovf, tmp, E);
    __syncthreads();
    for (int i = tid; i <= E; i += blockDim.x) offsets[E + 1 + i] = tmp[i];
    if (tid == 0 && tmp[E] > 0) report(status, 0u, MOE_CNT_OVERFLOW_ROWS, tmp[E]);
  }
}

__global__ void __launch_bounds__(kPermWarps * 32)
    scatter_kernel(int S, int d, int E, int K, int capacity, int tok_per_chunk, const int32_t* __restrict__ topk_idx,
                   const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets,
                   int32_t* __restrict__ row_of_slot, int32_t* __restrict__ token_of_row) {
  extern __shared__ int32_t sm[];
  int32_t* whist = sm;                        // [kPermWarps][E] per-warp counts, then bases
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int t0 = blockIdx.x * tok_per_chunk;
  const int t1 = min(S, t0 + tok_per_chunk);
  const int64_t s0 = static_cast<int64_t>(t0) * K;
  const int nslots = (t1 - t0) * K;
  const int per_warp = (nslots + kPermWarps - 1) / kPermWarps;
  const int w0 = warp * per_warp, w1 = min(nslots, w0 + per_warp);

  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  // pass 1: per-warp expert counts over the warp's contiguous slot range
  for (int b = w0; b < w1; b += 32) {
    const int s = b + lane;
    const bool act = s < w1;
    int e = act ? topk_idx[s0 + s] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(kFull, e);
    if (e >= 0 && lane == __ffs(peers) - 1) whist[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // bases: chunk base of the expert + counts of the warps before this one
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[static_cast<int64_t>(blockIdx.x) * E + e];
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = whist[w * E + e];
      whist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 2: ranks -> rows
  for (int b = w0; b < w1; b += 32) {
    const int s = b + lane;
    const bool act = s < w1;
    int e = act ? topk_idx[s0 + s] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(kFull, e);
    int row = -1;
    if (e >= 0) {
      const unsigned lt = (1u << lane) - 1u;
      const int r = whist[warp * E + e] + __popc(peers & lt);
      if (capacity <= 0)
        row = offsets[e] + r;
      else
        row = r < capacity ? e * capacity + r : E * capacity + offsets[E + 1 + e] + (r - capacity);
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) whist[warp * E + e] += __popc(peers);
    if (act) {
      row_of_slot[s0 + s] = row;
      if (row >= 0) token_of_row[row] = static_cast<int32_t>((s0 + s) / K);
    }
    __syncwarp();
  }
}

// Row gather: one warp per token reads its row once (16-byte vectors) and
// writes it to each of its K rows.  The grid grows with S, so the copy is
// spread over every SM.
template <typename T>
__global__ void __launch_bounds__(kPermWarps * 32)
    gather_rows_kernel(int S, int d, int K, const int32_t* __restrict__ row_of_slot, const T* __restrict__ x,
                       T* __restrict__ x_perm) {
  const int t = blockIdx.x * kPermWarps + (threadIdx.x >> 5);
  if (t >= S) return;
  const int lane = lane_id();
  const int my_row = lane < K ? __ldg(row_of_slot + static_cast<int64_t>(t) * K + lane) : -1;
  constexpr int V = Vec16<T>::N;
  const int nvec = d / V;
  const T* src = x + static_cast<int64_t>(t) * d;
#pragma unroll 2
  for (int base = 0; base < nvec; base += 32) {
    const int v = base + lane;
    const bool act = v < nvec;
    const uint4 val = act ? ldg16(src + v * V) : make_uint4(0, 0, 0, 0);
    for (int k = 0; k < K; ++k) {
      const int row = __shfl_sync(kFull, my_row, k);
      if (act && row >= 0) stg16(x_perm + static_cast<int64_t>(row) * d + v * V, val);
    }
  }
}

// Group table of the grouped GEMMs from the offsets: one group per expert
// (rows offsets[e] ..), or with a capacity two per expert, its primary rows
// (e*C ..) then its overflow rows (E*C + overflow offset ..), so that the
// overflow pass runs in the same launches right behind the expert's primary
// tiles while its weight tiles are still in L2; the shared expert last.
__device__ __forceinline__ void write_groups(int S, int E, int K, int capacity, int num_shared,
                                             const int32_t* offsets, GroupEntry* g1) {
  const int64_t R = capacity > 0 ? static_cast<int64_t>(E) * capacity + static_cast<int64_t>(S) * K
                                 : static_cast<int64_t>(S) * K;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int cnt = offsets[e + 1] - offsets[e];
    if (capacity <= 0) {
      g1[e] = GroupEntry{offsets[e], offsets[e], cnt, e};
    } else {
      const int prim = min(cnt, capacity);
      g1[2 * e] = GroupEntry{e * capacity, e * capacity, prim, e};
      const int orow = E * capacity + offsets[E + 1 + e];
      g1[2 * e + 1] = GroupEntry{orow, orow, cnt - prim, e};
    }
  }
  const int gs = capacity > 0 ? 2 * E : E;
  if (threadIdx.x == 0 && num_shared > 0) g1[gs] = GroupEntry{0, static_cast<int32_t>(R), S, E};
}


// Small batches (decode): histogram, scans, stable ranks, row maps and the
// group tables in one CTA -- the same counting sort as the chunked path with
// the whole slot range as one chunk split over 32 warps.
// sm: kSmallWarps * E + 3 * E + 1 ints of shared memory.
__device__ void permute_small_body(int S, int E, int K, int capacity, int num_shared, const int32_t* idx,
                                   int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* token_of_row,
                                   int64_t num_rows, GroupEntry* g1, StatusBlock* status, int32_t* sm) {
  int32_t* whist = sm;                      // [32][E]
  int32_t* cnt = sm + kSmallWarps * E;      // [E]
  int32_t* ovf = cnt + E;                   // [E]
  int32_t* tmp = ovf + E;                   // [E+1]
  __shared__ int32_t offs_s[2 * 257];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int nslots = S * K;
  const int per_warp = (nslots + kSmallWarps - 1) / kSmallWarps;
  const int w0 = warp * per_warp, w1 = min(nslots, w0 + per_warp);
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) whist[i] = 0;
  if (capacity > 0)
    for (int64_t r = threadIdx.x; r < num_rows; r += blockDim.x) token_of_row[r] = -1;
  __syncthreads();
  int bad = 0;
  for (int b = w0; b < w1; b += 32) {
    const int sl = b + lane;
    const bool act = sl < w1;
    int e = act ? idx[sl] : -1;
    if (act && (e < 0 || e >= E)) ++bad;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(kFull, e);
    if (e >= 0 && lane == __ffs(peers) - 1) whist[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  if (bad) report(status, MOE_STATUS_BAD_EXPERT_ID, MOE_CNT_BAD_ID, bad);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kSmallWarps; ++w) {
      const int c = whist[w * E + e];
      whist[w * E + e] = run;
      run += c;
    }
    cnt[e] = run;
    counts[e] = run;
    ovf[e] = capacity > 0 ? max(run - capacity, 0) : 0;
  }
  __syncthreads();
  warp0_exclusive_scan(cnt, tmp, E);
  __syncthreads();
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    offsets[i] = tmp[i];
    offs_s[i] = tmp[i];
  }
  if (capacity > 0) {
    __syncthreads();
    warp0_exclusive_scan(ovf, tmp, E);
    __syncthreads();
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
      offsets[E + 1 + i] = tmp[i];
      offs_s[E + 1 + i] = tmp[i];
    }
    if (threadIdx.x == 0 && tmp[E] > 0) report(status, 0u, MOE_CNT_OVERFLOW_ROWS, tmp[E]);
  }
  __syncthreads();
  for (int b = w0; b < w1; b += 32) {
    const int sl = b + lane;
    const bool act = sl < w1;
    int e = act ? idx[sl] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(kFull, e);
    int row = -1;
    if (e >= 0) {
      const int r = whist[warp * E + e] + __popc(peers & ((1u << lane) - 1u));
      if (capacity <= 0)
        row = offs_s[e] + r;
      else
        row = r < capacity ? e * capacity + r : E * capacity + offs_s[E + 1 + e] + (r - capacity);
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) whist[warp * E + e] += __popc(peers);
    if (act) {
      row_of_slot[sl] = row;
      if (row >= 0) token_of_row[row] = sl / K;
    }
    __syncwarp();
  }
  if (g1 != nullptr) write_groups(S, E, K, capacity, num_shared, offs_s, g1);
}

// x / x_perm (optional): the row gather of a tiny batch folded in -- every
// token row (row_chunks 16-byte pieces) copied to its slots' rows once the
// maps are written, so a decode step spends no launch on it.
__global__ void __launch_bounds__(kSmallWarps * 32)
    permute_small_kernel(int S, int E, int K, int capacity, int num_shared, const int32_t* topk_idx,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ row_of_slot, int32_t* __restrict__ token_of_row, int64_t num_rows,
                         GroupEntry* __restrict__ g1, StatusBlock* status, const uint4* __restrict__ x,
                         uint4* __restrict__ x_perm, int row_chunks) {
  extern __shared__ int32_t sm[];
  pdl_wait();
  pdl_trigger();
  permute_small_body(S, E, K, capacity, num_shared, topk_idx, counts, offsets, row_of_slot, token_of_row, num_rows,
                     g1, status, sm);
  if (x == nullptr) return;
  __syncthreads();  // the row maps written above are read back below
  const int64_t n = static_cast<int64_t>(S) * K * row_chunks;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const int64_t sl = i / row_chunks, c = i - sl * row_chunks;
    const int row = row_of_slot[sl];
    if (row >= 0) x_perm[static_cast<int64_t>(row) * row_chunks + c] = x[(sl / K) * row_chunks + c];
  }
}

// Row gather for small batches: one CTA per token, its threads split the row.
template <typename T>
__global__ void __launch_bounds__(256)
    gather_rows_cta_kernel(int d, int K, const int32_t* __restrict__ row_of_slot, const T* __restrict__ x,
                           T* __restrict__ x_perm) {
  __shared__ int32_t rows[32];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  if (threadIdx.x < K) rows[threadIdx.x] = row_of_slot[static_cast<int64_t>(t) * K + threadIdx.x];
  __syncthreads();
  constexpr int V = Vec16<T>::N;
  const int nvec = d / V;
  const T* src = x + static_cast<int64_t>(t) * d;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const uint4 val = ldg16(src + v * V);
    for (int k = 0; k < K; ++k)
      if (rows[k] >= 0) stg16(x_perm + static_cast<int64_t>(rows[k]) * d + v * V, val);
  }
}

__global__ void build_groups_kernel(int S, int E, int K, int capacity, int num_shared,
                                    const int32_t* __restrict__ offsets, GroupEntry* __restrict__ g1) {
  write_groups(S, E, K, capacity, num_shared, offsets, g1);
}

#ifdef MOE_DEBUG
__global__ void __launch_bounds__(256)
    debug_check_permutation_kernel(int S, int E, int K, int capacity, const int32_t* counts, const int32_t* offsets,
                                   const int32_t* row_of_slot, const int32_t* token_of_row, int64_t num_rows,
                                   StatusBlock* status) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  bool bad = false;
  if (tid < E) {
    const int c = counts[tid];
    if (c < 0 || offsets[tid + 1] - offsets[tid] != c) bad = true;
    if (capacity > 0) {
      const int ovf = c > capacity ? c - capacity : 0;
      if (offsets[E + 1 + tid + 1] - offsets[E + 1 + tid] != ovf) bad = true;
    }
  }
  if (tid == 0 && offsets[0] != 0) bad = true;
  for (int64_t sl = tid; sl < static_cast<int64_t>(S) * K; sl += nthreads) {
    const int r = row_of_slot[sl];
    if (r < -1 || r >= num_rows) {
      bad = true;
    } else if (r >= 0 && token_of_row[r] != static_cast<int32_t>(sl / K)) {
      bad = true;
    }
  }
  if (bad) report(status, MOE_STATUS_DEBUG_CHECK, -1);
}
#endif

}  // namespace

cudaError_t launch_debug_check_permutation(int S, int E, int K, int capacity, const int32_t* counts,
                                           const int32_t* offsets, const int32_t* row_of_slot,
                                           const int32_t* token_of_row, int64_t num_rows, StatusBlock* status,
                                           cudaStream_t stream) {
#ifdef MOE_DEBUG
  if (S <= 0) return cudaSuccess;
  const int64_t work = static_cast<int64_t>(S) * K > E ? static_cast<int64_t>(S) * K : E;
  const int blocks = static_cast<int>(work / 256 + 1 < 1184 ? work / 256 + 1 : 1184);
  debug_check_permutation_kernel<<<blocks, 256, 0, stream>>>(S, E, K, capacity, counts, offsets, row_of_slot,
                                                              token_of_row, num_rows, status);
  return cudaGetLastError();
#else
  (void)S; (void)E; (void)K; (void)capacity; (void)counts; (void)offsets; (void)row_of_slot; (void)token_of_row;
  (void)num_rows; (void)status; (void)stream;
  return cudaSuccess;
#endif
}

int permute_tokens_per_chunk(int K) { return K >= kChunkSlots ? 1 : kChunkSlots / K; }

int permute_num_chunks(int S, int K) {
  const int tpc = permute_tokens_per_chunk(K);
  return (S + tpc - 1) / tpc;
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t stream) {
  if (a.S == 0) {
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, stream);
    if (err == cudaSuccess)
      err = cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1) * (a.capacity > 0 ? 2 : 1), stream);
    if (err == cudaSuccess && a.num_rows > 0)
      err = cudaMemsetAsync(a.token_of_row, 0xFF, sizeof(int32_t) * a.num_rows, stream);
    return err;
  }
  cudaError_t err;
  const int64_t row_bytes = static_cast<int64_t>(a.d) * (a.act_dtype == MOE_BF16 ? 2 : 4);
  bool gathered = false;
  if (static_cast<int64_t>(a.S) * a.K <= kSmallSlots) {
    const size_t smem = sizeof(int32_t) * (kSmallWarps * a.E + 3 * a.E + 1);
    // tiny batches: the one CTA also copies the rows (a few hundred KB at most)
    gathered = a.x != nullptr && a.x_perm != nullptr && static_cast<int64_t>(a.S) * a.K * row_bytes <= kFoldGatherBytes;
    err = launch_pdl(permute_small_kernel, dim3(1), dim3(kSmallWarps * 32), smem, stream, a.S, a.E, a.K, a.capacity,
                     a.num_shared, a.topk_idx, a.counts, a.offsets, a.row_of_slot, a.token_of_row, a.num_rows, a.g1,
                     a.status, gathered ? static_cast<const uint4*>(a.x) : nullptr,
                     gathered ? static_cast<uint4*>(a.x_perm) : nullptr, static_cast<int>(row_bytes / 16));
    if (err != cudaSuccess || (err = cudaGetLastError()) != cudaSuccess) return err;
  } else {
    const int tpc = permute_tokens_per_chunk(a.K);
    const int nch = permute_num_chunks(a.S, a.K);
    if (a.capacity > 0) {
      // unused primary rows keep token -1
      err = cudaMemsetAsync(a.token_of_row, 0xFF, sizeof(int32_t) * a.num_rows, stream);
      if (err != cudaSuccess) return err;
    }
    count_kernel<<<nch, 256, sizeof(int32_t) * a.E, stream>>>(a.S, a.E, a.K, tpc, a.topk_idx, a.chunk_hist,
                                                                a.status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int scan_threads = 1024;
    const size_t scan_smem = sizeof(int32_t) * ((scan_threads / a.E) * a.E + 3 * a.E + 1);
    scan_kernel<<<1, scan_threads, scan_smem, stream>>>(a.E, nch, a.capacity, a.chunk_hist, a.counts, a.offsets,
                                                         a.status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const size_t smem = sizeof(int32_t) * kPermWarps * a.E;
    scatter_kernel<<<nch, kPermWarps * 32, smem, stream>>>(a.S, a.d, a.E, a.K, a.capacity, tpc, a.topk_idx,
                                                            a.chunk_hist, a.offsets, a.row_of_slot, a.token_of_row);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (a.g1 != nullptr) {
      build_groups_kernel<<<1, 256, 0, stream>>>(a.S, a.E, a.K, a.capacity, a.num_shared, a.offsets, a.g1);
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
  }
  if (a.x == nullptr || a.x_perm == nullptr || gathered) return cudaSuccess;
  if (a.S <= 256) {
#define MOE_GATHER_CTA(T)                                                                                    \
  err = launch_pdl(gather_rows_cta_kernel<T>, dim3(a.S), dim3(256), 0, stream, a.d, a.K,                       \
                   static_cast<const int32_t*>(a.row_of_slot), static_cast<const T*>(a.x), static_cast<T*>(a.x_perm))
    if (a.act_dtype == MOE_BF16)
      MOE_GATHER_CTA(__nv_bfloat16);
    else
      MOE_GATHER_CTA(float);
#undef MOE_GATHER_CTA
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  const int gblocks = (a.S + kPermWarps - 1) / kPermWarps;
  if (a.act_dtype == MOE_BF16)
    gather_rows_kernel<__nv_bfloat16><<<gblocks, kPermWarps * 32, 0, stream>>>(
        a.S, a.d, a.K, a.row_of_slot, static_cast<const __nv_bfloat16*>(a.x), static_cast<__nv_bfloat16*>(a.x_perm));
  else
    gather_rows_kernel<float><<<gblocks, kPermWarps * 32, 0, stream>>>(
        a.S, a.d, a.K, a.row_of_slot, static_cast<const float*>(a.x), static_cast<float*>(a.x_perm));
  return cudaGetLastError();
}

cudaError_t launch_build_groups(int S, int E, int K, int capacity, int num_shared, const int32_t* offsets,
                                GroupEntry* g1, StatusBlock* status, cudaStream_t stream) {
  (void)status;
  build_groups_kernel<<<1, 256, 0, stream>>>(S, E, K, capacity, num_shared, offsets, g1);
  return cudaGetLastError();
}

}  // namespace moe
