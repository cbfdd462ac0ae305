// moe_permute_static: the histogram / scan / permutation of moe_permute for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a runtime whose whole device-memory
// budget is fixed when it starts, code that runs inside an allocator or
// another callback where a nested cudaMalloc/cudaFree is not allowed, or a
// latency-critical loop that must not risk the device-wide synchronisation
// cudaFree can cause.  They cannot hand moe_permute a workspace, so this entry
// point keeps its only scratch -- the per-chunk expert histograms -- in a
// fixed-size array of device memory that belongs to the library itself.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (256 KB) until the process exits.  Host code cannot use
// the array's name as a device address, so the address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call made on it; make that first call before any stream capture.
// All calls share the one array and it keeps the last call's contents; the
// kernels overwrite every entry they read, so nothing needs clearing.  Calls
// that overlap on the GPU (different streams, or different host threads
// without ordering) race on the array.  Data problems are not reported
// through a status block here: an out-of-range expert id gets row -1.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace {

// Capacity of the built-in scratch: number of chunks x experts, int32 each.
constexpr int kStaticHistEntries = 65536;  // 256 KB

__device__ __align__(256) int32_t g_permute_hist[kStaticHistEntries];

// Device address of g_permute_hist on the current device (looked up once per
// device ordinal; returns nullptr if the lookup fails).  Host threads may make
// their first calls concurrently: each cache entry is an atomic pointer, and
// a thread that finds it empty looks the address up itself (every thread gets
// the same value for a device, so the relaxed store of either one is right).
int32_t* static_hist_for_current_device() {
  static std::atomic<int32_t*> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) {
    int32_t* known = cache[dev].load(std::memory_order_relaxed);
    if (known != nullptr) return known;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_hist) != cudaSuccess || p == nullptr) return nullptr;
  if (dev >= 0 && dev < 64) cache[dev].store(static_cast<int32_t*>(p), std::memory_order_relaxed);
  return static_cast<int32_t*>(p);
}

}  // namespace

extern "C" moe_status moe_permute_static(const moe_desc* desc, const void* x, const int32_t* topk_idx,
                                         int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                                         int32_t* token_of_row, void* x_perm, void* stream) {
  size_t unused = 0;
  const moe_status s = moe_workspace_size(desc, &unused);  // validates the descriptor
  if (s != MOE_OK) return s;
  if (counts == nullptr || offsets == nullptr || row_of_slot == nullptr || token_of_row == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (desc->num_tokens > 0 && topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (x && ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x_perm) & 15)))
    return MOE_ERR_INVALID_ARG;
  const int64_t entries =
      static_cast<int64_t>(moe::permute_num_chunks(desc->num_tokens, desc->top_k)) * desc->num_experts;
  if (entries > kStaticHistEntries) return MOE_ERR_WORKSPACE;  // more than the built-in scratch holds
  int32_t* hist = static_hist_for_current_device();
  if (hist == nullptr) return MOE_ERR_CUDA;
  moe::PermuteArgs a{};
  a.S = desc->num_tokens;
  a.d = desc->d_model;
  a.E = desc->num_experts;
  a.K = desc->top_k;
  a.capacity = desc->capacity;
  a.act_dtype = desc->act_dtype;
  a.topk_idx = topk_idx;
  a.chunk_hist = hist;
  a.counts = counts;
  a.offsets = offsets;
  a.row_of_slot = row_of_slot;
  a.token_of_row = token_of_row;
  a.x = x;
  a.x_perm = x_perm;
  a.num_rows = moe_routed_rows(desc);
  a.status = nullptr;
  return moe::launch_permute(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
