// Per-row E4M3 quantisation of bf16 activation rows, the activation half of
// the W8A8 expert path.
//
// ybb.press "MoE 推理工程深层实战" 3.3 lists FP8 (E4M3) as the production
// format for expert weights.  Running the expert GEMMs on 8-bit activations
// as well needs one scale per activation row; the reading used here:
//
//     s   = amax_j |x_j| / 448          (float32 division; 1 for an all-zero
//                                        row or a row holding a NaN)
//     q_j = E4M3_rn_satfinite(x_j / s)  (float32 division, then round to
//                                        nearest even, saturate at +-448,
//                                        NaN -> 0x7F)
//
// so that x_j ~= q_j * s, and the GEMM epilogue multiplies each accumulator
// row by its s.  One warp per row, two passes over the row (max, then
// encode; the second pass mostly hits L1/L2), 16-byte loads of 8 bf16 and
// 8-byte stores of 8 codes.
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
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kWarps = 8;  // rows per CTA

__device__ __forceinline__ uint8_t e4m3_code(float v) {
  if (isnan(v)) return 0x7F;
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// Row scale of d bf16 values (d % 8 == 0), computed by the calling warp.
__device__ __forceinline__ float row_scale_e4m3(const __nv_bfloat16* __restrict__ src, int d, int lane) {
  float amax = 0.0f;
  bool nan = false;
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8];
    bf16x8_to_f32(ldg16(src + c), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      amax = fmaxf(amax, fabsf(f[j]));
      nan |= isnan(f[j]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  nan = __any_sync(0xFFFFFFFFu, nan);
  return (!nan && amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// E4M3 codes of 8 bf16 values for the row scale s, packed in memory order.
__device__ __forceinline__ uint2 encode8_e4m3(const uint4& w, float s) {
  float f[8];
  bf16x8_to_f32(w, f);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    lo |= static_cast<uint32_t>(e4m3_code(__fdiv_rn(f[j], s))) << (8 * j);
    hi |= static_cast<uint32_t>(e4m3_code(__fdiv_rn(f[4 + j], s))) << (8 * j);
  }
  return make_uint2(lo, hi);
}

// Two-term codes: the row's multiplier 2^k (0 for a row with a non-finite
// value) and its scale 2^-k (NaN for such a row), computed by the calling warp.
__device__ __forceinline__ float row_pow2_e4m3(const __nv_bfloat16* __restrict__ src, int d, int lane,
                                               float* scale) {
  float amax = 0.0f;
  bool bad = false;
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8];
    bf16x8_to_f32(ldg16(src + c), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      amax = fmaxf(amax, fabsf(f[j]));
      bad |= !isfinite(f[j]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad) {
    *scale = __int_as_float(0x7FC00000);
    return 0.0f;
  }
  int k = 0;
  if (amax > 0.0f) {
    int ex;
    const float f = frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
    k = (f <= 0.875f ? 9 : 8) - ex;     // 448 = 0.875 * 2^9
    k = max(-126, min(126, k));
  }
  *scale = __int_as_float((127 - k) << 23);
  return __int_as_float((127 + k) << 23);
}

__device__ __forceinline__ float e4m3_value(uint8_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3)));
}

// Two-term codes of 8 bf16 values for the multiplier m, each term packed in memory order.
__device__ __forceinline__ void encode8_two_term(const uint4& w, float m, uint2& t1, uint2& t2) {
  float f[8];
  bf16x8_to_f32(w, f);
  uint32_t a[2] = {0, 0}, b[2] = {0, 0};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float v = f[j] * m;
    const uint8_t c1 = e4m3_code(v);
    const uint8_t c2 = e4m3_code(v - e4m3_value(c1));
    a[j >> 2] |= static_cast<uint32_t>(c1) << (8 * (j & 3));
    b[j >> 2] |= static_cast<uint32_t>(c2) << (8 * (j & 3));
  }
  t1 = make_uint2(a[0], a[1]);
  t2 = make_uint2(b[0], b[1]);
}

// Two-term codes of one row (d % 8 == 0): term 1 at dst[0, d), term 2 at dst[d, 2d).
__device__ __forceinline__ void two_term_row(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                                             float* __restrict__ scale, int d, int lane) {
  float sc;
  const float m = row_pow2_e4m3(src, d, lane, &sc);
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    uint2 t1, t2;
    encode8_two_term(ldg16(src + c), m, t1, t2);
    *reinterpret_cast<uint2*>(dst + c) = t1;
    *reinterpret_cast<uint2*>(dst + d + c) = t2;
  }
  if (lane == 0) *scale = sc;
}

// Quantise one row of d bf16 values (d % 8 == 0) with the calling warp.
__device__ __forceinline__ void quantize_row(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                                             float* __restrict__ scale, int d, int lane) {
  const float s = row_scale_e4m3(src, d, lane);
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) *reinterpret_cast<uint2*>(dst + c) = encode8_e4m3(ldg16(src + c), s);
  if (lane == 0) *scale = s;
}

// The permutation's row gather fused with the quantisation: a warp per
// token computes the token row's scale and codes once and writes them to the
// token's K rows of the expert-sorted buffer (row_of_slot; -1 = none), and to
// row t of q_x / s_x when given (the shared expert's operand).  TERMS = 1:
// W8A8 codes (rows of d bytes); TERMS = 2: two-term codes (rows of 2d bytes).
template <int TERMS>
__global__ void __launch_bounds__(kWarps * 32)
    gather_quantize_kernel(int S, int d, int K, const int32_t* __restrict__ row_of_slot,
                           const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ q_perm,
                           float* __restrict__ s_perm, uint8_t* __restrict__ q_x, float* __restrict__ s_x) {
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= S) return;
  const int lane = lane_id();
  const int my_row = lane < K ? __ldg(row_of_slot + static_cast<int64_t>(t) * K + lane) : -1;
  const __nv_bfloat16* src = x + static_cast<int64_t>(t) * d;
  const int64_t pitch = static_cast<int64_t>(TERMS) * d;
  float s = 1.0f, m = 1.0f;
  if (TERMS == 1)
    s = row_scale_e4m3(src, d, lane);
  else
    m = row_pow2_e4m3(src, d, lane, &s);
  for (int c = lane * 8; c < d; c += 256) {
    uint2 q, q2 = make_uint2(0, 0);
    if (TERMS == 1)
      q = encode8_e4m3(ldg16(src + c), s);
    else
      encode8_two_term(ldg16(src + c), m, q, q2);
    for (int k = 0; k < K; ++k) {
      const int row = __shfl_sync(0xFFFFFFFFu, my_row, k);
      if (row >= 0) {
        *reinterpret_cast<uint2*>(q_perm + row * pitch + c) = q;
        if (TERMS == 2) *reinterpret_cast<uint2*>(q_perm + row * pitch + d + c) = q2;
      }
    }
    if (q_x != nullptr) {
      *reinterpret_cast<uint2*>(q_x + t * pitch + c) = q;
      if (TERMS == 2) *reinterpret_cast<uint2*>(q_x + t * pitch + d + c) = q2;
    }
  }
  if (my_row >= 0) s_perm[my_row] = s;
  if (lane == 0 && s_x != nullptr) s_x[t] = s;
}

// Rows of a group table (groups != nullptr) or `single_rows` contiguous rows.
// The rows of all groups form one flat range (a prefix over the groups'
// row counts in shared memory); each warp takes rows of it with a grid
// stride, so the grid is sized by the rows there are, not by groups x the
// largest group.
constexpr int kQuantMaxGroups = 520;
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_kernel(const GroupEntry* __restrict__ groups, int num_groups, int use_out_rows, int shared_slab,
                         int64_t single_rows, const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                         float* __restrict__ scale, int64_t dst_rows, const __nv_bfloat16* __restrict__ src_sh,
                         uint8_t* __restrict__ dst_sh, float* __restrict__ scale_sh, int64_t sh_rows, int d,
                         int terms) {
  __shared__ int64_t start[kQuantMaxGroups + 1];
  const int lane = lane_id(), warp = threadIdx.x >> 5;
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
          const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
          if (lane >= off) incl += o;
        }
        if (g < num_groups) start[g] = carry + incl - rows;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (lane == 0) start[num_groups] = carry;
    }
    __syncthreads();
    total = start[num_groups];
  }
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kWarps + warp; i < total;
       i += static_cast<int64_t>(gridDim.x) * kWarps) {
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
    if (row < 0 || row >= (shared ? sh_rows : dst_rows)) continue;
    const __nv_bfloat16* in = shared ? src_sh + row * d : src + row * d;
    uint8_t* out = (shared ? dst_sh : dst) + row * terms * d;
    float* sc = (shared ? scale_sh : scale) + row;
    if (terms == 2)
      two_term_row(in, out, sc, d, lane);
    else
      quantize_row(in, out, sc, d, lane);
  }
}

}  // namespace

// Grid of the row quantisation: enough warps for `rows`, at most 16 CTAs per SM.
dim3 quantize_grid(int64_t rows) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  }
  const int64_t want = (rows + kWarps - 1) / kWarps;
  return dim3(static_cast<unsigned>(want < 16 * sms ? (want > 0 ? want : 1) : 16 * sms));
}

cudaError_t launch_quantize_rows(const void* src, uint8_t* dst, float* scale, int64_t rows, int d, int terms,
                                 cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (d <= 0 || d % 8 != 0 || (terms != 1 && terms != 2)) return cudaErrorInvalidValue;
  quantize_rows_kernel<<<quantize_grid(rows), kWarps * 32, 0, stream>>>(
      nullptr, 0, 0, -1, rows, static_cast<const __nv_bfloat16*>(src), dst, scale, rows, nullptr, nullptr, nullptr, 0,
      d, terms);
  return cudaGetLastError();
}

cudaError_t launch_gather_quantize(int S, int d, int K, const int32_t* row_of_slot, const void* x, uint8_t* q_perm,
                                   float* s_perm, uint8_t* q_x, float* s_x, int terms, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  if (d <= 0 || d % 8 != 0 || K < 1 || K > 32 || (terms != 1 && terms != 2)) return cudaErrorInvalidValue;
  const dim3 grid((S + kWarps - 1) / kWarps);
  if (terms == 2)
    gather_quantize_kernel<2><<<grid, kWarps * 32, 0, stream>>>(S, d, K, row_of_slot,
                                                                 static_cast<const __nv_bfloat16*>(x), q_perm,
                                                                 s_perm, q_x, s_x);
  else
    gather_quantize_kernel<1><<<grid, kWarps * 32, 0, stream>>>(S, d, K, row_of_slot,
                                                                 static_cast<const __nv_bfloat16*>(x), q_perm,
                                                                 s_perm, q_x, s_x);
  return cudaGetLastError();
}

cudaError_t launch_quantize_group_rows(const GroupEntry* groups, int num_groups, int use_out_rows, int shared_slab,
                                       const void* src, uint8_t* dst, float* scale, int64_t dst_rows,
                                       const void* src_shared, uint8_t* dst_shared, float* scale_shared,
                                       int64_t shared_rows, int d, int64_t max_total_rows, int terms,
                                       cudaStream_t stream) {
  if (num_groups <= 0 || max_total_rows <= 0) return cudaSuccess;
  if (num_groups > kQuantMaxGroups || d <= 0 || d % 8 != 0 || (terms != 1 && terms != 2))
    return cudaErrorInvalidValue;
  quantize_rows_kernel<<<quantize_grid(max_total_rows), kWarps * 32, 0, stream>>>(
      groups, num_groups, use_out_rows, shared_slab, 0, static_cast<const __nv_bfloat16*>(src), dst, scale, dst_rows,
      static_cast<const __nv_bfloat16*>(src_shared), dst_shared, scale_shared, shared_rows, d, terms);
  return cudaGetLastError();
}

}  // namespace moe
