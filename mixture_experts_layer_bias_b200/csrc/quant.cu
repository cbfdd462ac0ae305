// Per-row E4M3 codes of bf16 activation rows, for the expert GEMMs that run
// on the E4M3 tensor-core kind.
//
// ybb.press "MoE 推理工程深层实战" 3.3 lists FP8 (E4M3) as the production
// format for expert weights.  Two ways of feeding the activations:
//
// W8A8 (one term).  Running the expert GEMMs on 8-bit activations as well
// needs one scale per activation row; the reading used here:
//
//     s   = amax_j |x_j| / 448          (float32 division; 1 for an all-zero
//                                        row or a row holding a NaN)
//     q_j = E4M3_rn_satfinite(x_j / s)  (float32 division, then round to
//                                        nearest even, saturate at +-448,
//                                        NaN -> 0x7F)
//
// so that x_j ~= q_j * s, and the GEMM epilogue multiplies each accumulator
// row by its s.
//
// Two-term codes (E4M3 weights with bf16 activations).  The tensor cores
// have no bf16 x E4M3 product, so a bf16 row is written as two E4M3 terms
// that the GEMM multiplies with the stored weight codes in two f8f6f4 MMAs
// accumulating into one fp32 sum:
//
//     k    = the largest integer with amax * 2^k <= 448 (k = 0 for an
//            all-zero row), clamped to [-126, 126]
//     v_j  = x_j * 2^k                    (exact: a power-of-two scaling)
//     c1_j = E4M3_rn(v_j),  c2_j = E4M3_rn(v_j - c1_j)   (the difference is
//            exact in float32)
//     row scale = 2^-k
//
// A bf16 value has 8 significant bits and c1 keeps the leading 4 (with
// rounding), so the remainder has at most 4 and c1 + c2 = v exactly unless
// the remainder falls below the E4M3 subnormal spacing 2^-9, i.e. unless
// |v_j| < 0.25 (|x_j| below about amax * 2^-10.8); there the error is at
// most 2^-10 in v, 2^-17.8 * amax in x.  A row holding an infinity or a NaN
// gets the scale NaN, so its outputs are NaN.
//
// Layout of the work: a row is read twice (max, then codes; the second read
// mostly hits L1/L2) by a warp, or, when there are few rows (decode), by a
// whole CTA so that the row's loads spread over 8 warps.  Codes are made two
// at a time by the paired float -> E4M3 conversion, and the value of c1 is
// recovered with integer and float arithmetic (below), so the conversion unit
// sees one instruction per two codes of each term.
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "pdl.cuh"
#include "row_coding.cuh"

namespace moe {

namespace {

using namespace coding;
constexpr int kWarps = coding::kCodeWarps;  // warps per CTA
constexpr unsigned kFull = 0xFFFFFFFFu;

// The permutation's row gather fused with the coding: token t's row is coded
// once (by a warp, or by the CTA with T = 256) and the codes go to the
// token's K rows of the expert-sorted buffer (row_of_slot; -1 = none), and to
// row t of q_x / s_x when given (the shared expert's operand).  Rows of
// terms * d codes.
template <int T>
__global__ void __launch_bounds__(kWarps * 32)
    gather_quantize_kernel(int S, int d, int K, int terms, const int32_t* __restrict__ row_of_slot,
                           const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ q_perm,
                           float* __restrict__ s_perm, uint8_t* __restrict__ q_x, float* __restrict__ s_x) {
  const int per_cta = kWarps * 32 / T;
  const int t = blockIdx.x * per_cta + static_cast<int>(threadIdx.x) / T;
  const int tid = static_cast<int>(threadIdx.x) % T;
  pdl_wait();
  pdl_trigger();
  if (t >= S) return;  // T = 256: the whole CTA leaves together
  __shared__ int rows[kWarps][32];
  int* my_rows = rows[threadIdx.x >> 5];
  if (T == 32) {
    if (tid < K) my_rows[tid] = __ldg(row_of_slot + static_cast<int64_t>(t) * K + tid);
    __syncwarp();
  } else {
    if (tid < K) rows[0][tid] = __ldg(row_of_slot + static_cast<int64_t>(t) * K + tid);
    my_rows = rows[0];
    __syncthreads();
  }
  const __nv_bfloat16* src = x + static_cast<int64_t>(t) * d;
  const int64_t pitch = static_cast<int64_t>(terms) * d;
  RowPieces<T> rp;
  float amax, s, m;
  bool nan, nonfinite;
  row_load_amax<T>(src, d, tid, rp, amax, nan, nonfinite);
  row_scale(terms, amax, nan, nonfinite, s, m);
  auto put = [&](const uint4& w, int c) {
    uint2 q, q2 = make_uint2(0, 0);
    if (terms == 2)
      encode8_two_term(w, m, q, q2);
    else
      q = encode8_w8a8(w, s);
    for (int k = 0; k < K; ++k) {
      const int row = my_rows[k];
      if (row >= 0) {
        *reinterpret_cast<uint2*>(q_perm + row * pitch + c) = q;
        if (terms == 2) *reinterpret_cast<uint2*>(q_perm + row * pitch + d + c) = q2;
      }
    }
    if (q_x != nullptr) {
      *reinterpret_cast<uint2*>(q_x + t * pitch + c) = q;
      if (terms == 2) *reinterpret_cast<uint2*>(q_x + t * pitch + d + c) = q2;
    }
  };
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int c = (tid + i * T) * 8;
    if (c < d) put(rp.v[i], c);
  }
  for (int c = (tid + kVec * T) * 8; c < d; c += T * 8) put(ldg16(src + c), c);
  if (tid < K && my_rows[tid] >= 0) s_perm[my_rows[tid]] = s;
  if (tid == 0 && s_x != nullptr) s_x[t] = s;
}

// Rows of a group table (groups != nullptr) or `single_rows` contiguous rows.
// The rows of all groups form one flat range (a prefix over the groups'
// row counts in shared memory); each warp (T = 32) or CTA (T = 256) takes
// rows of it with a grid stride, so the grid is sized by the rows there are,
// not by groups x the largest group.
constexpr int kQuantMaxGroups = 520;
template <int T>
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_kernel(const GroupEntry* __restrict__ groups, int num_groups, int use_out_rows, int shared_slab,
                         int64_t single_rows, const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                         float* __restrict__ scale, int64_t dst_rows, const __nv_bfloat16* __restrict__ src_sh,
                         uint8_t* __restrict__ dst_sh, float* __restrict__ scale_sh, int64_t sh_rows, int d,
                         int terms) {
  __shared__ int64_t start[kQuantMaxGroups + 1];
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  int64_t total = single_rows;
  if (groups != nullptr) {
    if (warp == 0) {
      int64_t carry = 0;
      for (int base = 0; base < num_groups; base += 32) {
        const int g = base + lane;
        const int64_t rows = g < num_groups ? max(groups[g].rows, 0) : 0;
        int64_t incl = rows;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int64_t o = __shfl_up_sync(kFull, incl, off);
          if (lane >= off) incl += o;
        }
        if (g < num_groups) start[g] = carry + incl - rows;
        carry += __shfl_sync(kFull, incl, 31);
      }
      if (lane == 0) start[num_groups] = carry;
    }
    __syncthreads();
    total = start[num_groups];
  }
  const int per_cta = kWarps * 32 / T;
  const int tid = static_cast<int>(threadIdx.x) % T;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * per_cta + static_cast<int>(threadIdx.x) / T; i < total;
       i += static_cast<int64_t>(gridDim.x) * per_cta) {
    int64_t row;
    bool shared = false;
    if (groups == nullptr) {
      row = i;
    } else {
      int lo = 0, hi = num_groups;  // start[lo] <= i < start[lo + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (start[mid] <= i)
          lo = mid;
        else
          hi = mid;
      }
      const GroupEntry g = groups[lo];
      shared = g.expert == shared_slab && src_sh != nullptr;
      row = (shared ? 0 : (use_out_rows ? g.out_row0 : g.a_row0)) + (i - start[lo]);
    }
    // rows outside the buffers (a corrupt table) are skipped; the GEMM reports the group
    // (uniform over the T threads of the row, so a CTA row never splits at its barriers)
    if (row < 0 || row >= (shared ? sh_rows : dst_rows)) continue;
    const __nv_bfloat16* in = shared ? src_sh + row * d : src + row * d;
    uint8_t* out = (shared ? dst_sh : dst) + row * terms * d;
    float* sc = (shared ? scale_sh : scale) + row;
    code_row<T>(in, out, sc, d, terms, tid);
  }
}

// 1-D bulk copy global -> shared of `bytes` (a multiple of 16, both addresses
// 16-byte aligned), completion counted on `bar` in bytes.  No multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Many rows of at most kStagedMaxCols columns: each CTA codes chunks of
// `chunk` consecutive rows of the flat row range.  Warp 0 stages a chunk's
// rows in shared memory by bulk copies (one per row), into one of two chunk
// buffers, so the next chunk streams in while the warps code this one (a row
// per warp: max, then codes, both from shared memory).  The waits on the
// copies are bounded; a CTA that gives up reports MOE_STATUS_TIMEOUT, lets its
// copies in flight land (bounded again) and exits.
constexpr int kStagedMaxCols = 4096;
constexpr int kMaxChunk = 32;
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_staged_kernel(const GroupEntry* __restrict__ groups, int num_groups, int use_out_rows,
                                int shared_slab, int64_t single_rows, const __nv_bfloat16* __restrict__ src,
                                uint8_t* __restrict__ dst, float* __restrict__ scale, int64_t dst_rows,
                                const __nv_bfloat16* __restrict__ src_sh, uint8_t* __restrict__ dst_sh,
                                float* __restrict__ scale_sh, int64_t sh_rows, int d, int terms, int chunk,
                                StatusBlock* status) {
  extern __shared__ __align__(128) uint8_t stage[];  // [2][chunk][d] bf16
  __shared__ int64_t start[kQuantMaxGroups + 1];
  __shared__ __align__(8) uint64_t full[2];
  __shared__ int64_t row_of[2][kMaxChunk];  // staged row -> its row in src / src_sh (-1: none)
  __shared__ int8_t sh_of[2][kMaxChunk];    // 1: the shared expert's row (src_sh)
  __shared__ int fail;
  __shared__ int issued[2];                 // parity + 1 of the last copies into each buffer, 0: none
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fail = 0;
    issued[0] = issued[1] = 0;
    fence_mbar_init();
  }
  pdl_wait();
  pdl_trigger();
  int64_t total = single_rows;
  if (groups != nullptr && warp == 0) {
    int64_t carry = 0;
    for (int base = 0; base < num_groups; base += 32) {
      const int g = base + lane;
      const int64_t rows = g < num_groups ? max(groups[g].rows, 0) : 0;
      int64_t incl = rows;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < num_groups) start[g] = carry + incl - rows;
      carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) start[num_groups] = carry;
  }
  __syncthreads();
  if (groups != nullptr) total = start[num_groups];
  const int64_t nchunks = (total + chunk - 1) / chunk;
  const uint32_t row_bytes = static_cast<uint32_t>(d) * 2;
  uint32_t phase[2] = {0, 0};
  int abort_flag = 0;
  // warp 0: rows of chunk c into buffer b
  auto issue = [&](int64_t c, int b) {
    int n_valid = 0;
    for (int r = lane; r < chunk; r += 32) {
      const int64_t i = c * chunk + r;
      int64_t row = -1;
      int sh = 0;
      if (i < total) {
        if (groups == nullptr) {
          row = i;
        } else {
          int lo = 0, hi = num_groups;  // start[lo] <= i < start[lo + 1]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (start[mid] <= i)
              lo = mid;
            else
              hi = mid;
          }
          const GroupEntry g = groups[lo];
          sh = g.expert == shared_slab && src_sh != nullptr;
          row = (sh ? 0 : (use_out_rows ? g.out_row0 : g.a_row0)) + (i - start[lo]);
        }
        // rows outside the buffers (a corrupt table) are skipped; the GEMM reports the group
        if (row < 0 || row >= (sh ? sh_rows : dst_rows)) row = -1;
      }
      row_of[b][r] = row;
      sh_of[b][r] = static_cast<int8_t>(sh);
      n_valid += row >= 0;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n_valid += __shfl_xor_sync(kFull, n_valid, off);
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[b], static_cast<uint32_t>(n_valid) * row_bytes);
      issued[b] = static_cast<int>(phase[b]) + 1;
    }
    __syncwarp();
    for (int r = lane; r < chunk; r += 32) {
      const int64_t row = row_of[b][r];
      if (row >= 0)
        bulk_load(stage + (static_cast<size_t>(b) * chunk + r) * row_bytes, (sh_of[b][r] ? src_sh : src) + row * d,
                  row_bytes, &full[b]);
    }
  };
  int b = 0;
  int64_t c = blockIdx.x;
  if (warp == 0 && c < nchunks) issue(c, 0);
  for (; c < nchunks; c += gridDim.x) {
    const int64_t cn = c + gridDim.x;
    if (warp == 0 && cn < nchunks) issue(cn, b ^ 1);  // released by the barrier ending the previous chunk
    if (!mbar_wait(&full[b], phase[b], &abort_flag)) atomicOr(&fail, 1);
    __syncthreads();
    if (fail) break;
    if (threadIdx.x == 0) issued[b] = 0;
    phase[b] ^= 1u;
    for (int r = warp; r < chunk; r += kWarps) {
      const int64_t row = row_of[b][r];
      if (row < 0) continue;
      const bool sh = sh_of[b][r];
      const uint8_t* rs = stage + (static_cast<size_t>(b) * chunk + r) * row_bytes;
      uint32_t acc = 0;
      for (int col = lane * 8; col < d; col += 256)
        acc = absmax_bits8(acc, *reinterpret_cast<const uint4*>(rs + col * 2));
      const uint32_t bits = __reduce_max_sync(kFull, max(acc & 0xFFFFu, acc >> 16));
      float sc, mult;
      row_scale(terms, __uint_as_float(bits << 16), bits > 0x7F80u, bits >= 0x7F80u, sc, mult);
      uint8_t* out = (sh ? dst_sh : dst) + row * terms * d;
      for (int col = lane * 8; col < d; col += 256)
        code_piece(*reinterpret_cast<const uint4*>(rs + col * 2), out, d, col, terms, sc, mult);
      if (lane == 0) (sh ? scale_sh : scale)[row] = sc;
    }
    __syncthreads();  // buffer b is free again
    b ^= 1;
  }
  if (fail && threadIdx.x == 0) {
    report(status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
    // copies still in flight must land before the CTA's shared memory goes away
    int never = 0;
    for (int i = 0; i < 2; ++i)
      if (issued[i]) mbar_wait(&full[i], static_cast<uint32_t>(issued[i] - 1), &never);
  }
}

// Per-device host caches (atomics: host threads may launch concurrently).
constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  return dev;
}

int device_sms() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  int sms = dev < kMaxDevices ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (sms <= 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    if (dev < kMaxDevices) cache[dev].store(sms, std::memory_order_relaxed);
  }
  return sms;
}

// A CTA per row when there are few rows (up to four per SM: decode) or rows
// too long for a warp to hold in registers; otherwise a warp per row.
bool cta_rows(int64_t rows, int d) {
  return rows <= 4 * static_cast<int64_t>(device_sms()) || d > 32 * 8 * kVec;
}

// Grid of the row coding: enough warps (or CTAs) for `rows`, at most 16 CTAs per SM.
dim3 quantize_grid(int64_t rows, int d) {
  const int64_t per_cta = cta_rows(rows, d) ? 1 : kWarps;
  const int64_t want = (rows + per_cta - 1) / per_cta;
  const int64_t cap = 16 * static_cast<int64_t>(device_sms());
  return dim3(static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap));
}

cudaError_t launch_rows(const GroupEntry* groups, int num_groups, int use_out_rows, int shared_slab,
                        int64_t single_rows, const void* src, uint8_t* dst, float* scale, int64_t dst_rows,
                        const void* src_sh, uint8_t* dst_sh, float* scale_sh, int64_t sh_rows, int d, int terms,
                        int64_t max_rows, StatusBlock* status, cudaStream_t stream) {
  const auto* s = static_cast<const __nv_bfloat16*>(src);
  const auto* ss = static_cast<const __nv_bfloat16*>(src_sh);
  if (!cta_rows(max_rows, d) && d <= kStagedMaxCols) {
    // staged chunks: a multiple of 8 rows (one per warp), about 24 KB per chunk buffer (two per CTA)
    const int chunk = std::min(kMaxChunk, std::max(kWarps, (12288 / d) / kWarps * kWarps));
    const size_t smem = static_cast<size_t>(2) * chunk * d * 2;
    // the largest dynamic shared memory enabled so far, per device (the attribute is per device)
    static std::atomic<size_t> attr_bytes[kMaxDevices];
    const int dev = current_device();
    if (dev >= kMaxDevices || smem > attr_bytes[dev].load(std::memory_order_relaxed)) {
      cudaError_t e = cudaFuncSetAttribute(quantize_rows_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      if (dev < kMaxDevices) {
        size_t cur = attr_bytes[dev].load(std::memory_order_relaxed);
        while (smem > cur && !attr_bytes[dev].compare_exchange_weak(cur, smem, std::memory_order_relaxed)) {
        }
      }
    }
    const int64_t chunks = (max_rows + chunk - 1) / chunk;
    // as many CTAs as are resident at once (shared memory, 8 CTAs of 256 threads at most)
    const int per_sm = static_cast<int>(std::max<size_t>(1, std::min<size_t>(8, 232448 / (smem + 6144))));
    const int64_t cap = static_cast<int64_t>(per_sm) * device_sms();
    const dim3 grid(static_cast<unsigned>(chunks < cap ? chunks : cap));
    cudaError_t e = launch_pdl(quantize_rows_staged_kernel, grid, dim3(kWarps * 32), smem, stream, groups, num_groups,
                               use_out_rows, shared_slab, single_rows, s, dst, scale, dst_rows, ss, dst_sh, scale_sh,
                               sh_rows, d, terms, chunk, status);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const dim3 grid = quantize_grid(max_rows, d);
  cudaError_t e;
  if (cta_rows(max_rows, d))
    e = launch_pdl(quantize_rows_kernel<kWarps * 32>, grid, dim3(kWarps * 32), 0, stream, groups, num_groups,
                   use_out_rows, shared_slab, single_rows, s, dst, scale, dst_rows, ss, dst_sh, scale_sh, sh_rows, d,
                   terms);
  else
    e = launch_pdl(quantize_rows_kernel<32>, grid, dim3(kWarps * 32), 0, stream, groups, num_groups, use_out_rows,
                   shared_slab, single_rows, s, dst, scale, dst_rows, ss, dst_sh, scale_sh, sh_rows, d, terms);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_rows(const void* src, uint8_t* dst, float* scale, int64_t rows, int d, int terms,
                                 cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (d <= 0 || d % 8 != 0 || (terms != 1 && terms != 2)) return cudaErrorInvalidValue;
  return launch_rows(nullptr, 0, 0, -1, rows, src, dst, scale, rows, nullptr, nullptr, nullptr, 0, d, terms, rows,
                     nullptr, stream);
}

cudaError_t launch_gather_quantize(int S, int d, int K, const int32_t* row_of_slot, const void* x, uint8_t* q_perm,
                                   float* s_perm, uint8_t* q_x, float* s_x, int terms, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  if (d <= 0 || d % 8 != 0 || K < 1 || K > 32 || (terms != 1 && terms != 2)) return cudaErrorInvalidValue;
  const auto* xs = static_cast<const __nv_bfloat16*>(x);
  cudaError_t e;
  if (cta_rows(S, d))
    e = launch_pdl(gather_quantize_kernel<kWarps * 32>, dim3(S), dim3(kWarps * 32), 0, stream, S, d, K, terms,
                   row_of_slot, xs, q_perm, s_perm, q_x, s_x);
  else
    e = launch_pdl(gather_quantize_kernel<32>, dim3((S + kWarps - 1) / kWarps), dim3(kWarps * 32), 0, stream, S, d, K,
                   terms, row_of_slot, xs, q_perm, s_perm, q_x, s_x);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quantize_group_rows(const GroupEntry* groups, int num_groups, int use_out_rows, int shared_slab,
                                       const void* src, uint8_t* dst, float* scale, int64_t dst_rows,
                                       const void* src_shared, uint8_t* dst_shared, float* scale_shared,
                                       int64_t shared_rows, int d, int64_t max_total_rows, int terms,
                                       StatusBlock* status, cudaStream_t stream) {
  if (num_groups <= 0 || max_total_rows <= 0) return cudaSuccess;
  if (num_groups > kQuantMaxGroups || d <= 0 || d % 8 != 0 || (terms != 1 && terms != 2))
    return cudaErrorInvalidValue;
  return launch_rows(groups, num_groups, use_out_rows, shared_slab, 0, src, dst, scale, dst_rows, src_shared,
                     dst_shared, scale_shared, shared_rows, d, terms, max_total_rows, status, stream);
}

}  // namespace moe
