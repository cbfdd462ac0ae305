// Pieces shared by the tensor-core grouped GEMM kernel: launch parameters,
// group lookup, the device-side split-K choice, the split-K finalize kernel
// and tensor-map encoding.
#pragma once

#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace gemm {

constexpr int kMaxGroups = 520;  // 2 x 256 experts (primary + overflow) + shared

struct TcParams {
  const GroupEntry* groups;  // nullptr: one group of `single_rows` rows, slab 0
  int single_rows;
  int num_groups;
  int shared_slab;
  int a_rows_from_out;
  int num_slabs;
  int n_per_slab;
  int N, K;
  int bn_out;   // output columns per tile (128 SwiGLU, 256 otherwise)
  int n_tiles;  // ceil(N / bn_out)
  int64_t out_rows;
  const float* bias;
  const float* scale0;
  const float* scale1;
  void* out;
  int out_f32;
  int max_ksplit;      // 1 = no split-K
  float* partial;      // fp32 [max_ksplit][out_rows][pcols] (split-K partial sums)
  int pcols;           // 2N (SwiGLU: gate then up) or N
  int* ksplit_out;     // the split chosen on the device (read by the finalize kernel)
  int test_stall;      // test hook: the producer delivers nothing (the bounded waits must give up)
  int a_terms;         // E4M3 activations: 1, or 2 for two-term codes (A rows of 2K codes, term 2 at column K)
  int a_pack;          // two-term codes, 64-row m-blocks: both terms in one M=128 MMA (A rows 0.., 64..)
  int bm;              // rows of an m-block: 128, or 64 when no group exceeds 128 rows
  int tma_out;         // 1: the output tensor map is valid (full 32-row quarters use bulk tensor stores)
  const float* row_scale;         // E4M3 activations: per-row scale of the A operand rows (nullptr: none)
  const float* row_scale_shared;  // ... of the shared expert's A rows (indexed by row within the group)
  StatusBlock* status;
};

// Scale of A row `r` (within group `g`) for 8-bit activations, 1 otherwise.
__device__ __forceinline__ float a_row_scale(const TcParams& p, const GroupEntry& g, int r) {
  if (p.row_scale == nullptr) return 1.0f;
  if (g.expert == p.shared_slab && p.row_scale_shared != nullptr) return __ldg(p.row_scale_shared + r);
  return __ldg(p.row_scale + (p.a_rows_from_out ? g.out_row0 : g.a_row0) + r);
}

__device__ __forceinline__ GroupEntry group_at(const TcParams& p, int g) {
  if (p.groups == nullptr) return GroupEntry{0, 0, p.single_rows, 0};
  return p.groups[g];
}

// Split-K factor for `tiles` output tiles on `grid` persistent CTAs: the
// split that minimises the busiest CTA's work, counted in K-blocks plus one
// K-block's worth of fixed cost per work unit (its epilogue), with >= 4
// K-blocks per unit; ties to the smaller split.
__device__ __forceinline__ int choose_ksplit(int tiles, int grid, int nk, int kmax) {
  if (tiles <= 0 || kmax <= 1) return 1;
  constexpr int kUnitCost = 1;
  int best = 1;
  int64_t best_cost = static_cast<int64_t>((tiles + grid - 1) / grid) * (nk + kUnitCost);
  for (int ks = 2; ks <= kmax; ++ks) {
    if (nk / ks < 4) break;
    const int64_t units = static_cast<int64_t>(tiles) * ks;
    const int64_t cost = ((units + grid - 1) / grid) * ((nk + ks - 1) / ks + kUnitCost);
    if (cost < best_cost) {
      best = ks;
      best_cost = cost;
    }
  }
  return best;
}

__device__ __forceinline__ bool group_ok(const GroupEntry& g, const TcParams& p) {
  return g.rows > 0 && g.expert >= 0 && g.expert < p.num_slabs && g.out_row0 >= 0 &&
         static_cast<int64_t>(g.out_row0) + g.rows <= p.out_rows && g.a_row0 >= 0;
}

// Split-K: every epilogue warp of a CTA owns one region of its tile (32 rows
// of one TMEM lane quarter x half of the tile's columns) and, per split, writes
// its raw fp32 accumulators there to the split's slice of the partial buffer.
// splitk_finalize_kernel then sums the slices in split order (deterministic
// whatever the order the CTAs ran in), applies the epilogue and stores the
// output: one thread per four output columns of a row, so many rows are
// reduced in parallel.

// Epilogue of split-K sums: gate/up sums g, u (SwiGLU) or sums v, with the
// row scale rs, channel scales and bias of column n + j.
template <int EPI>
__device__ __forceinline__ float splitk_out(const TcParams& p, int64_t sbase, int n, int j, float g, float u,
                                            float rs) {
  float gv = g * rs;
  if (p.scale0 != nullptr) gv *= p.scale0[sbase + n + j];
  if (EPI == EPI_SWIGLU) {
    float uv = u * rs;
    if (p.scale1 != nullptr) uv *= p.scale1[sbase + n + j];
    return gv / (1.0f + __expf(-gv)) * uv;
  }
  if (EPI == EPI_GELU_BIAS || EPI == EPI_BIAS) gv += p.bias[sbase + n + j];
  if (EPI == EPI_GELU_BIAS) gv = 0.5f * gv * (1.0f + erff(gv * 0.70710678118654752f));
  return gv;
}

// Sums of the ks slices of the float4 at `src` and, with TWO, of the float4
// at `src + off` (slice stride `slice`), each in split order; up to eight
// slices of each are loaded before their sums, so that all loads of a batch
// are in flight together.  Read at L2 (ld.global.cg): other CTAs wrote them.
template <bool TWO>
__device__ __forceinline__ void splitk_sums4(const float* src, int64_t off, int64_t slice, int ks, float4& g,
                                             float4& u) {
  g = make_float4(0.f, 0.f, 0.f, 0.f);
  u = g;
  for (int s = 0; s < ks; s += 8) {
    float4 a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (s + i < ks) {
        a[i] = __ldcg(reinterpret_cast<const float4*>(src + (s + i) * slice));
        if (TWO) b[i] = __ldcg(reinterpret_cast<const float4*>(src + off + (s + i) * slice));
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (s + i < ks) {
        g.x += a[i].x; g.y += a[i].y; g.z += a[i].z; g.w += a[i].w;
        if (TWO) {
          u.x += b[i].x; u.y += b[i].y; u.z += b[i].z; u.w += b[i].w;
        }
      }
    }
  }
}

// Split-K finalize: for every valid row of every group, sum the partial slices
// in split order and apply the epilogue; one thread per four output columns.
// Exits at once when the GEMM ran without a split.  Launched under
// programmatic dependent launch: it waits for the GEMM before reading.
template <int EPI>
__global__ void __launch_bounds__(256) splitk_finalize_kernel(TcParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int ks = *p.ksplit_out;
  if (ks <= 1) return;
  const GroupEntry grp = group_at(p, blockIdx.z);
  const int r = blockIdx.y;
  if (r >= grp.rows || grp.expert < 0 || grp.expert >= p.num_slabs) return;
  const int n = (blockIdx.x * 256 + threadIdx.x) * 4;
  const int N = p.N;
  if (n >= N) return;
  const int64_t orow = static_cast<int64_t>(grp.out_row0) + r;
  if (orow >= p.out_rows) return;
  const int64_t sbase = static_cast<int64_t>(grp.expert) * N;
  const int64_t slice = p.out_rows * static_cast<int64_t>(p.pcols);
  const float rs = a_row_scale(p, grp, r);
  const float* src = p.partial + orow * p.pcols + n;
  float4 g, u;
  splitk_sums4<EPI == EPI_SWIGLU>(src, N, slice, ks, g, u);
  float o[4];
  o[0] = splitk_out<EPI>(p, sbase, n, 0, g.x, u.x, rs);
  o[1] = splitk_out<EPI>(p, sbase, n, 1, g.y, u.y, rs);
  o[2] = splitk_out<EPI>(p, sbase, n, 2, g.z, u.z, rs);
  o[3] = splitk_out<EPI>(p, sbase, n, 3, g.w, u.w, rs);
  if (p.out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * N + n) = make_float4(o[0], o[1], o[2], o[3]);
  } else {
    const uint2 packed = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + orow * N + n) = packed;
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D map over [rows][k] (row-major) of bf16 (elem_bytes 2) or 8-bit (1)
// elements; box = one 128-byte swizzle row of k by box_rows rows.
// 2-D map over an output [rows][cols] (row-major, bf16 or fp32) for bulk
// tensor stores of 32 x 32 element boxes, no swizzle.
inline bool make_store_map(CUtensorMap* m, void* base, int64_t rows, int cols, int elem_bytes) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr || rows <= 0 || cols <= 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (static_cast<int64_t>(cols) * elem_bytes) % 16 != 0) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool make_map(CUtensorMap* m, const void* base, int64_t rows, int k, int box_rows = 128, int elem_bytes = 2) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr || rows <= 0 || k <= 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (static_cast<int64_t>(k) * elem_bytes) % 16 != 0) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k) * elem_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


}  // namespace gemm
}  // namespace moe
