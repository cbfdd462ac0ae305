// fp32 grouped expert GEMM on CUDA cores (exact fp32 products and sums).
//
// Used for fp32 layers such as the tiny GeLU workload, whose 1e-4 relative
// tolerance rules out tf32/bf16 tensor-core math.  Expert FFN of jsqmd.com
// "第11章 MoE模型推理" 11.1.2: E_i(x) = GeLU(x W1 + b1) W2 + b2, run as one
// launch per projection over all expert groups (grid z = group).
//
// Tile 32 rows x 64 output columns, K-chunks of 32 staged in shared memory;
// 256 threads, 2 x 4 outputs each.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmArgs a) {
  __shared__ float as[32][33];
  __shared__ float bs[64][33];
  const GroupEntry grp = a.groups[blockIdx.z];
  const int m0 = blockIdx.y * 32;
  if (m0 >= grp.rows) return;
  const int n0 = blockIdx.x * 64;
  const int N = a.N, K = a.K;
  const bool shared_a = grp.expert == a.shared_slab;
  const float* A = static_cast<const float*>(shared_a ? a.a_shared : a.a);
  const int64_t arow0 = (a.a_rows_from_out ? grp.out_row0 : grp.a_row0) + m0;
  const float* B = static_cast<const float*>(a.b0) + static_cast<int64_t>(grp.expert) * a.n_per_slab * K;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[2][4] = {};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = tid; i < 32 * 32; i += 256) {
      const int r = i >> 5, c = i & 31;
      as[r][c] = (m0 + r < grp.rows && k0 + c < K) ? A[(arow0 + r) * K + k0 + c] : 0.0f;
    }
    for (int i = tid; i < 64 * 32; i += 256) {
      const int r = i >> 5, c = i & 31;
      bs[r][c] = (n0 + r < N && k0 + c < K) ? B[static_cast<int64_t>(n0 + r) * K + k0 + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const float a0 = as[ty * 2][c], a1 = as[ty * 2 + 1][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float b = bs[tx * 4 + j][c];
        acc[0][j] = fmaf(a0, b, acc[0][j]);
        acc[1][j] = fmaf(a1, b, acc[1][j]);
      }
    }
    __syncthreads();
  }
  float* out = static_cast<float*>(a.out);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = m0 + ty * 2 + i;
    if (r >= grp.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (a.scale0 != nullptr) v *= a.scale0[static_cast<int64_t>(grp.expert) * N + n];
      if (EPI == EPI_GELU_BIAS || EPI == EPI_BIAS) v += a.bias[static_cast<int64_t>(grp.expert) * N + n];
      if (EPI == EPI_GELU_BIAS) v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
      out[static_cast<int64_t>(grp.out_row0 + r) * N + n] = v;
    }
  }
}

}  // namespace

// grid.y covers the largest possible group (a token picks an expert at most
// once, so no group has more than S rows).
cudaError_t launch_grouped_gemm_f32(const GemmArgs& a, cudaStream_t stream) {
  const int64_t max_rows = a.max_group_rows;
  if (max_rows == 0 || a.num_groups == 0) return cudaSuccess;
  dim3 grid((a.N + 63) / 64, static_cast<unsigned>((max_rows + 31) / 32), a.num_groups);
  switch (a.epilogue) {
    case EPI_GELU_BIAS: gemm_f32_kernel<EPI_GELU_BIAS><<<grid, 256, 0, stream>>>(a); break;
    case EPI_BIAS: gemm_f32_kernel<EPI_BIAS><<<grid, 256, 0, stream>>>(a); break;
    case EPI_NONE: gemm_f32_kernel<EPI_NONE><<<grid, 256, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moe
