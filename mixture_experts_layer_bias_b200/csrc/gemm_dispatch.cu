// Grouped GEMM launch parameters: fills the parameter block of the
// tensor-core kernel from the launch arguments (split-K budget, epilogue
// operands, output mode) and hands it to the token-rows kernel launcher.
#include <stdlib.h>
#include <string.h>

#include "gemm_common.cuh"

namespace moe {

using namespace gemm;

#ifdef MOE_B200_TEST_HOOKS
// Failure-detection test hook, compiled only into the test build of the
// library (libmoe_b200_testhooks.so): moe_test_stall_gemms(n) makes the next
// n GEMM launches run with a producer that delivers nothing, so every bounded
// wait of those launches gives up and reports MOE_STATUS_TIMEOUT.
namespace {
int g_stall_budget = 0;
int take_test_stall() {
  if (g_stall_budget <= 0) return 0;
  --g_stall_budget;
  return 1;
}
}  // namespace
extern "C" void moe_test_stall_gemms(int n) { g_stall_budget = n > 0 ? n : 0; }
#endif

cudaError_t launch_grouped_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  if (a.num_groups <= 0 || a.num_groups > kMaxGroups) return cudaErrorInvalidValue;
  if (a.groups == nullptr && (a.num_groups != 1 || a.max_total_rows > INT32_MAX)) return cudaErrorInvalidValue;
  TcParams p;
  p.groups = a.groups;
  p.single_rows = a.groups == nullptr ? static_cast<int>(a.max_total_rows) : 0;
  p.num_groups = a.num_groups;
  p.shared_slab = a.shared_slab;
  p.a_rows_from_out = a.a_rows_from_out;
  p.n_per_slab = a.n_per_slab;
  p.num_slabs = static_cast<int>(a.b_rows / a.n_per_slab);
  p.N = a.N;
  p.K = a.K;
  p.bn_out = a.epilogue == EPI_SWIGLU ? 128 : 256;
  p.n_tiles = (a.N + p.bn_out - 1) / p.bn_out;
  p.out_rows = a.out_rows;
  p.bias = a.bias;
  p.scale0 = a.scale0;
  p.scale1 = a.scale1;
  p.out = a.out;
  p.out_f32 = a.out_f32;
  p.status = a.status;
  p.pcols = a.epilogue == EPI_SWIGLU ? 2 * a.N : a.N;
  p.partial = a.partial;
  p.ksplit_out = a.ksplit_out;
  p.max_ksplit = 1;
  if (a.partial != nullptr && a.ksplit_out != nullptr && a.partial_bytes > 0) {
    // as many K slices as the partial buffer holds for every output row
    const int64_t per_split = a.out_rows * static_cast<int64_t>(p.pcols) * 4;
    p.max_ksplit = static_cast<int>(per_split > 0 ? a.partial_bytes / per_split : 1);
    if (p.max_ksplit > 16) p.max_ksplit = 16;
    if (p.max_ksplit < 1) p.max_ksplit = 1;
  }
#ifdef MOE_B200_TEST_HOOKS
  p.test_stall = take_test_stall();
#else
  p.test_stall = 0;
#endif
  p.tma_out = 0;  // set by the launcher when it can map the output
  p.a_terms = 1;  // set by the launcher
  p.a_pack = 0;
  p.bm = 128;  // set by the launcher
  p.row_scale = a.fp8 ? a.row_scale : nullptr;
  p.row_scale_shared = a.fp8 ? a.row_scale_shared : nullptr;
  if (a.fp8 && a.row_scale == nullptr) return cudaErrorInvalidValue;
  return launch_grouped_gemm_single(a, p, num_sms, stream);
}

}  // namespace moe
