// Grouped GEMM dispatch: fills the launch parameters shared by the tensor-core
// kernels and picks one of them (token rows as M, the default; weights as M
// on one CTA; weights as M on a CTA pair).  E4M3 operands always take the
// token-rows kernel.
#include <stdlib.h>
#include <string.h>

#include "gemm_common.cuh"

namespace moe {

using namespace gemm;

namespace {

// Test hook for the failure-detection tests: MOE_B200_TEST_STALL_GEMM=n makes
// the next n one-CTA GEMM launches of this process run with a producer that
// delivers nothing, so their bounded waits give up and report
// MOE_STATUS_TIMEOUT.  Unset (the default) it costs nothing.
int take_test_stall() {
  static int budget = -1;
  if (budget < 0) {
    const char* v = getenv("MOE_B200_TEST_STALL_GEMM");
    budget = v != nullptr ? atoi(v) : 0;
    if (budget < 0) budget = 0;
  }
  if (budget == 0) return 0;
  --budget;
  return 1;
}

// Kernel choice (read once): MOE_B200_GEMM=pair or =wt selects the CTA-pair or
// the one-CTA weights-as-M kernel, =hybrid the weights-as-M kernel for all but
// the SwiGLU up projection, =pairtok the token-rows kernel on CTA pairs for
// large groups; otherwise (or =single) the one-CTA token-rows kernel.
int gemm_kernel_choice() {
  static int choice = -1;
  if (choice < 0) {
    const char* v = getenv("MOE_B200_GEMM");
    choice = 0;
    if (v != nullptr && strcmp(v, "pair") == 0) choice = 1;
    if (v != nullptr && strcmp(v, "wt") == 0) choice = 2;
    if (v != nullptr && strcmp(v, "hybrid") == 0) choice = 3;
    if (v != nullptr && strcmp(v, "single") == 0) choice = 4;
    if (v != nullptr && strcmp(v, "pairtok") == 0) choice = 5;
  }
  return choice;
}

}  // namespace

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
  p.test_stall = 0;
  p.tma_out = 0;  // set by the token-rows launcher when it can map the output
  p.row_scale = a.fp8 ? a.row_scale : nullptr;
  p.row_scale_shared = a.fp8 ? a.row_scale_shared : nullptr;
  if (a.fp8 && a.row_scale == nullptr) return cudaErrorInvalidValue;
  const int choice = a.fp8 ? 0 : gemm_kernel_choice();  // 8-bit operands: token-rows kernel only
  if (choice == 1) return launch_grouped_gemm_pair(a, p, num_sms, stream);
  p.test_stall = take_test_stall();
  if (choice == 2 || (choice == 3 && a.epilogue != EPI_SWIGLU)) return launch_grouped_gemm_wt(a, p, num_sms, stream);
  return launch_grouped_gemm_single(a, p, num_sms, stream, choice == 4 ? 1 : (choice == 5 ? 2 : 0));
}

}  // namespace moe
