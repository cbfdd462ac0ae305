// Sliding-window expert load and the aux-loss-free selection-bias update.
//
// ybb.press "MoE 推理工程深层实战" 2.3: DeepSeek-V3-style routing adds a bias to
// the selection keys and recomputes it from a sliding-window token count
// over a window of 1000 tokens, steering the routing distribution
// without gradients.  The page does not print the update rule; the one used
// here moves each expert's bias against its deviation from the mean load:
//
//     b_e <- b_e + gamma * sign(mean - count_e)        (float32)
//
// where count_e is the number of (token, k) slots routed to e among the last
// `window` tokens and mean = tokens_in_window * K / E.
//
// State (caller-owned device memory, zeroed by moe_bias_state_init):
//   int32 header {filled, head}, int32 counts[E], int32 ring[window][K]
// The ring holds the expert ids of the last `window` tokens, filled from
// position 0; a batch of S tokens takes the next S positions (only its last
// `window` tokens when S >= window), decrementing the counts of the tokens it
// replaces.  One CTA does the whole update: the batch's count changes are
// integer shared-memory atomics, so the result does not depend on their order.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(1024)
    bias_update_kernel(int S, int E, int K, int W, const int32_t* __restrict__ topk_idx, float gamma,
                       int32_t* __restrict__ hdr, int32_t* __restrict__ counts, int32_t* __restrict__ ring,
                       float* __restrict__ sel_bias, int32_t* __restrict__ out_counts) {
  __shared__ int32_t delta[256];  // count changes of this batch (E <= 256), shared-memory atomics
  const int filled = hdr[0], head = hdr[1];
  for (int e = threadIdx.x; e < E; e += blockDim.x) delta[e] = 0;
  __syncthreads();
  int new_filled, new_head;
  if (S >= W) {
    for (int64_t s = threadIdx.x; s < static_cast<int64_t>(W) * K; s += blockDim.x) {
      const int64_t src = static_cast<int64_t>(S - W) * K + s;  // the batch's last W tokens
      const int id = topk_idx[src];
      const bool ok = id >= 0 && id < E;
      ring[s] = ok ? id : -1;
      if (ok) atomicAdd(&delta[id], 1);
    }
    new_filled = W;
    new_head = 0;
  } else {
    for (int64_t s = threadIdx.x; s < static_cast<int64_t>(S) * K; s += blockDim.x) {
      const int i = static_cast<int>(s / K), k = static_cast<int>(s % K);
      const int pos = (head + i) % W;
      const int64_t at = static_cast<int64_t>(pos) * K + k;
      if (filled == W || pos < filled) {
        const int old = ring[at];
        if (old >= 0 && old < E) atomicSub(&delta[old], 1);
      }
      const int id = topk_idx[s];
      const bool ok = id >= 0 && id < E;
      ring[at] = ok ? id : -1;
      if (ok) atomicAdd(&delta[id], 1);
    }
    new_filled = min(W, filled + S);
    new_head = (head + S) % W;
  }
  __syncthreads();
  const float mean = __fdiv_rn(static_cast<float>(new_filled * K), static_cast<float>(E));
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = (S >= W ? 0 : counts[e]) + delta[e];
    counts[e] = c;
    const float diff = __fsub_rn(mean, static_cast<float>(c));
    float b = sel_bias[e];
    if (diff > 0.0f)
      b = __fadd_rn(b, gamma);
    else if (diff < 0.0f)
      b = __fsub_rn(b, gamma);
    sel_bias[e] = b;
    if (out_counts != nullptr) out_counts[e] = c;
  }
  if (threadIdx.x == 0) {
    hdr[0] = new_filled;
    hdr[1] = new_head;
  }
}

}  // namespace

size_t bias_state_bytes(int E, int K, int window) {
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  return 256 + up(sizeof(int32_t) * E) + up(sizeof(int32_t) * static_cast<size_t>(window) * K);
}

cudaError_t launch_bias_update(int S, int E, int K, int window, const int32_t* topk_idx, float gamma, void* state,
                               float* sel_bias, int32_t* window_counts, cudaStream_t stream) {
  char* base = static_cast<char*>(state);
  int32_t* hdr = reinterpret_cast<int32_t*>(base);
  int32_t* counts = reinterpret_cast<int32_t*>(base + 256);
  int32_t* ring = reinterpret_cast<int32_t*>(base + 256 + ((sizeof(int32_t) * E + 255) & ~size_t(255)));
  bias_update_kernel<<<1, 1024, 0, stream>>>(S, E, K, window, topk_idx, gamma, hdr, counts, ring, sel_bias,
                                             window_counts);
  return cudaGetLastError();
}

}  // namespace moe
