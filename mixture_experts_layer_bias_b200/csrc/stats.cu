// Load report of one routing, computed on the device from the per-expert
// counts: max/mean expert load (jsqmd.com "第11章 MoE模型推理" 11.2.3), the
// standard deviation of the per-expert counts and the token drop rate
// (ybb.press "MoE 推理工程深层实战" 1.2, the table of inference metrics),
// rows above the capacity (2.2 of the same page, overflow buffering).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kStatsThreads = 256;  // one thread per expert (E <= 256)

__global__ void __launch_bounds__(kStatsThreads)
    load_stats_kernel(int E, int64_t slots, int capacity, const int32_t* __restrict__ counts, double* __restrict__ out) {
  __shared__ double red[kStatsThreads];
  __shared__ double sh_sum, sh_max, sh_over;
  const int e = threadIdx.x;
  const double c = e < E ? static_cast<double>(counts[e]) : 0.0;
  // sum, max and rows over capacity: tree reductions in a fixed order (deterministic)
  auto reduce = [&](double v, int op) {
    red[e] = v;
    __syncthreads();
    for (int s = kStatsThreads / 2; s >= 1; s >>= 1) {
      if (e < s) red[e] = op == 1 ? fmax(red[e], red[e + s]) : red[e] + red[e + s];
      __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
  };
  const double sum = reduce(c, 0);
  const double mx = reduce(e < E ? c : -1.0, 1);
  const double over = reduce(capacity > 0 ? fmax(c - capacity, 0.0) : 0.0, 0);
  if (e == 0) {
    sh_sum = sum;
    sh_max = mx;
    sh_over = over;
  }
  const double mean = static_cast<double>(slots) / E;
  const double dev = e < E ? c - mean : 0.0;
  const double var = reduce(dev * dev, 0) / E;
  if (e == 0) {
    out[MOE_LS_MAX_OVER_MEAN] = mean > 0.0 ? sh_max / mean : 0.0;
    out[MOE_LS_STD] = sqrt(var);
    out[MOE_LS_MEAN] = mean;
    out[MOE_LS_MAX] = sh_max;
    out[MOE_LS_OVERFLOW_ROWS] = sh_over;
    out[MOE_LS_DROPPED] = static_cast<double>(slots) - sh_sum;
  }
}

}  // namespace

cudaError_t launch_load_stats(int E, int64_t slots, int capacity, const int32_t* counts, double* out,
                              cudaStream_t stream) {
  load_stats_kernel<<<1, kStatsThreads, 0, stream>>>(E, slots, capacity, counts, out);
  return cudaGetLastError();
}

}  // namespace moe
