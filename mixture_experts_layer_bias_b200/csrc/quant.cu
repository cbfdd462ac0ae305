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
// row t of q_x / s_x when given (the shared expert's operand).
__global__ void __launch_bounds__(kWarps * 32)
    gather_quantize_kernel(int S, int d, int K, const int32_t* __restrict__ row_of_slot,
                           const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ q_perm,
                           float* __restrict__ s_perm, uint8_t* __restrict__ q_x, float* __restrict__ s_x) {
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= S) return;
  const int lane = lane_id();
  const int my_row = lane < K ? __ldg(row_of_slot + static_cast<int64_t>(t) * K + lane) : -1;
  const __nv_bfloat16* src = x + static_cast<int64_t>(t) * d;
  const float s = row_scale_e4m3(src, d, lane);
  for (int c = lane * 8; c < d; c += 256) {
    const uint2 q = encode8_e4m3(ldg16(src + c), s);
    for (int k = 0; k < K; ++k) {
      const int row = __shfl_sync(0xFFFFFFFFu, my_row, k);
      if (row >= 0) *reinterpret_cast<uint2*>(q_perm + static_cast<int64_t>(row) * d + c) = q;
    }
    if (q_x != nullptr) *reinterpret_cast<uint2*>(q_x + static_cast<int64_t>(t) * d + c) = q;
  }
  if (my_row >= 0) s_perm[my_row] = s;
  if (lane == 0 && s_x != nullptr) s_x[t] = s;
}

// Rows of a group table (groups != nullptr) or `single_rows` contiguous rows.
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_kernel(const GroupEntry* __restrict__ groups, int use_out_rows, int shared_slab,
                         int64_t single_rows, const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                         float* __restrict__ scale, int64_t dst_rows, const __nv_bfloat16* __restrict__ src_sh,
                         uint8_t* __restrict__ dst_sh, float* __restrict__ scale_sh, int64_t sh_rows, int d) {
  const int lane = lane_id();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  int64_t row;
  bool shared = false;
  if (groups == nullptr) {
    if (r >= single_rows) return;
    row = r;
  } else {
    const GroupEntry g = groups[blockIdx.y];
    if (r >= g.rows) return;
    shared = g.expert == shared_slab && src_sh != nullptr;
    row = (shared ? 0 : (use_out_rows ? g.out_row0 : g.a_row0)) + r;
  }
  // rows outside the buffers (a corrupt table) are skipped; the GEMM reports the group
  if (row < 0 || row >= (shared ? sh_rows : dst_rows)) return;
  if (shared)
    quantize_row(src_sh + row * d, dst_sh + row * d, scale_sh + row, d, lane);
  else
    quantize_row(src + row * d, dst + row * d, scale + row, d, lane);
}

}  // namespace

cudaError_t launch_quantize_rows(const void* src, uint8_t* dst, float* scale, int64_t rows, int d,
                                 cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > INT32_MAX || d <= 0 || d % 8 != 0) return cudaErrorInvalidValue;
  quantize_rows_kernel<<<dim3(static_cast<unsigned>(blocks)), kWarps * 32, 0, stream>>>(
      nullptr, 0, -1, rows, static_cast<const __nv_bfloat16*>(src), dst, scale, rows, nullptr, nullptr, nullptr, 0,
      d);
  return cudaGetLastError();
}

cudaError_t launch_gather_quantize(int S, int d, int K, const int32_t* row_of_slot, const void* x, uint8_t* q_perm,
                                   float* s_perm, uint8_t* q_x, float* s_x, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  if (d <= 0 || d % 8 != 0 || K < 1 || K > 32) return cudaErrorInvalidValue;
  gather_quantize_kernel<<<(S + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(
      S, d, K, row_of_slot, static_cast<const __nv_bfloat16*>(x), q_perm, s_perm, q_x, s_x);
  return cudaGetLastError();
}

cudaError_t launch_quantize_group_rows(const GroupEntry* groups, int num_groups, int use_out_rows, int shared_slab,
                                       const void* src, uint8_t* dst, float* scale, int64_t dst_rows,
                                       const void* src_shared, uint8_t* dst_shared, float* scale_shared,
                                       int64_t shared_rows, int d, int64_t max_group_rows, cudaStream_t stream) {
  if (num_groups <= 0 || max_group_rows <= 0) return cudaSuccess;
  const int64_t blocks = (max_group_rows + kWarps - 1) / kWarps;
  if (blocks > INT32_MAX || num_groups > 65535 || d <= 0 || d % 8 != 0) return cudaErrorInvalidValue;
  quantize_rows_kernel<<<dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(num_groups)), kWarps * 32, 0,
                         stream>>>(groups, use_out_rows, shared_slab, 0, static_cast<const __nv_bfloat16*>(src), dst,
                                   scale, dst_rows, static_cast<const __nv_bfloat16*>(src_shared), dst_shared,
                                   scale_shared, shared_rows, d);
  return cudaGetLastError();
}

}  // namespace moe
