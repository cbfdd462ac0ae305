// Gate-weighted combine back into token order, and the FP8 weight decode.
//
// jsqmd.com "第11章 MoE模型推理" 11.3.1 step 6 (weighted sum of the K expert
// outputs by the top-k probabilities) and 11.2.1 (outputs restored to the
// original token order); plumephp.com "MoE 混合专家推理", worked example:
// output = 0.55 * e0(x) + 0.30 * e3(x), normalised.
//
// One CTA per token; threads stride over 16-byte vectors of the d_model row;
// fp32 sums in k order, then the shared expert's row (gate 1), one rounding to
// the output type at the end.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "pdl.cuh"

namespace moe {

namespace {

// One CTA per token, its threads splitting the row (16-byte vectors): each
// thread issues the loads of all K rows of its vectors before the sums, so an
// SM keeps many rows in flight.  Launched under programmatic dependent launch.
template <typename T>
__global__ void __launch_bounds__(256)
    combine_cta_kernel(int d, int K, const T* __restrict__ y_perm, const int32_t* __restrict__ row_of_slot,
                       const float* __restrict__ topk_w, int64_t shared_row0, T* __restrict__ y, int64_t num_rows,
                       StatusBlock* status) {
  __shared__ int32_t rows[32];
  __shared__ float gates[32];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  if (threadIdx.x < K) {
    int r = row_of_slot[static_cast<int64_t>(t) * K + threadIdx.x];
#ifdef MOE_DEBUG
    if (r >= num_rows) {  // a row outside y_perm: report and skip it
      report(status, MOE_STATUS_DEBUG_CHECK, -1);
      r = -1;
    }
#endif
    rows[threadIdx.x] = r;
    gates[threadIdx.x] = topk_w[static_cast<int64_t>(t) * K + threadIdx.x];
  }
  __syncthreads();
  constexpr int V = Vec16<T>::N;
  const int nvec = d / V;
#pragma unroll 2
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.0f;
    for (int k = 0; k < K; ++k) {
      if (rows[k] < 0) continue;
      float f[V];
      unpack16<T>(ldg16(y_perm + static_cast<int64_t>(rows[k]) * d + v * V), f);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] = fmaf(gates[k], f[j], acc[j]);
    }
    if (shared_row0 >= 0) {
      float f[V];
      unpack16<T>(ldg16(y_perm + (shared_row0 + t) * d + v * V), f);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += f[j];
    }
    stg16(y + static_cast<int64_t>(t) * d + v * V, pack16<T>(acc));
  }
}

// 16 E4M3 codes -> 16 bf16 values (every E4M3 value is exact in f16 and in
// bf16, so both conversions are exact).
__global__ void dequant_e4m3_kernel(const uint4* __restrict__ q, uint4* __restrict__ out, int64_t n16) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(q + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((w[j] >> (16 * h)) & 0xFFFFu);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
        const __half2 hv = *reinterpret_cast<const __half2*>(&hr);
        const float2 f = __half22float2(hv);
        o[2 * j + h] = pack_bf16x2(f.x, f.y);
      }
    }
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  if (a.S == 0) return cudaSuccess;
  // threads per token: enough 16-byte vectors for each (d / 8 or d / 4 of them), at most 256
  const int nvec = a.act_dtype == MOE_BF16 ? a.d / 8 : a.d / 4;
  const int threads = nvec >= 256 ? 256 : (nvec >= 128 ? 128 : 64);
  cudaError_t err;
  if (a.act_dtype == MOE_BF16)
    err = launch_pdl(combine_cta_kernel<__nv_bfloat16>, dim3(a.S), dim3(threads), 0, stream, a.d, a.K,
                     static_cast<const __nv_bfloat16*>(a.y_perm), a.row_of_slot, a.topk_w, a.shared_row0,
                     static_cast<__nv_bfloat16*>(a.y), a.num_rows, a.status);
  else
    err = launch_pdl(combine_cta_kernel<float>, dim3(a.S), dim3(threads), 0, stream, a.d, a.K,
                     static_cast<const float*>(a.y_perm), a.row_of_slot, a.topk_w, a.shared_row0,
                     static_cast<float*>(a.y), a.num_rows, a.status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_dequant_e4m3(const uint8_t* q, void* out_bf16, int64_t n, cudaStream_t stream) {
  const int64_t n16 = n / 16;
  if (n16 == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (n16 + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  dequant_e4m3_kernel<<<blocks, threads, 0, stream>>>(reinterpret_cast<const uint4*>(q),
                                                      reinterpret_cast<uint4*>(out_bf16), n16);
  return cudaGetLastError();
}

}  // namespace moe
