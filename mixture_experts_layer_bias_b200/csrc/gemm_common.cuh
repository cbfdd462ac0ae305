// Pieces shared by the tensor-core grouped GEMM kernel: launch parameters,
// group lookup, the device-side split-K choice, the split-K reduction of the
// last-arriving slice and tensor-map encoding.
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
  int* tile_count;     // split-K arrival counters, kRegionsPerTile per tile, zero between launches
  int max_tiles;       // tiles the counters cover (more tiles: no split-K)
  int test_stall;      // test hook: the producer delivers nothing (the bounded waits must give up)
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
// smallest split whose work units fill the CTAs' waves clearly better
// (>= 5 points of wave efficiency per step up), with >= 4 K-blocks per unit.
__device__ __forceinline__ int choose_ksplit(int tiles, int grid, int nk, int kmax) {
  if (tiles <= 0 || kmax <= 1) return 1;
  auto eff = [&](int units) {
    const int waves = (units + grid - 1) / grid;
    return static_cast<float>(units) / static_cast<float>(waves * grid);
  };
  int best = 1;
  float best_eff = eff(tiles);
  for (int ks = 2; ks <= kmax; ++ks) {
    if (nk / ks < 4) break;
    const float e = eff(tiles * ks);
    if (e > best_eff + 0.05f) {
      best = ks;
      best_eff = e;
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
// One arrival counter per (tile, region) counts the slices written; the warp
// whose slice completes the count sums the region's slices in split order
// (deterministic whatever the arrival order), applies the epilogue and stores
// the output rows, then resets the counter for the next launch.
constexpr int kRegionsPerTile = 8;

// The last arriver's reduction of region (q, half) of tile `ti`: rows
// m_idx*128 + q*32 .. +31 of the group, lane j taking output columns
// n0 + 2j, n0 + 2j + 1 (SwiGLU, 64 columns per half: gate at n, up at N + n
// in the slices) or n0 + 4j .. n0 + 4j + 3 (128 columns per half).  Partial
// sums are read at L2 (ld.global.cg): other CTAs wrote them in this launch.
template <int EPI>
__device__ __forceinline__ void splitk_reduce_region(const TcParams& p, const GroupEntry& grp, int m_row0, int n_tile,
                                                     int ks, int half, int lane) {
  const int N = p.N;
  const int64_t slice = p.out_rows * static_cast<int64_t>(p.pcols);
  const int64_t sbase = static_cast<int64_t>(grp.expert) * N;
  const int r1 = min(m_row0 + 32, grp.rows);
  if (EPI == EPI_SWIGLU) {
    const int n = n_tile * p.bn_out + half * 64 + 2 * lane;
    if (n >= N) return;  // N is a multiple of 8, so n + 1 < N as well
    float c0[2] = {1.0f, 1.0f}, c1[2] = {1.0f, 1.0f};
    if (p.scale0 != nullptr) { c0[0] = p.scale0[sbase + n]; c0[1] = p.scale0[sbase + n + 1]; }
    if (p.scale1 != nullptr) { c1[0] = p.scale1[sbase + n]; c1[1] = p.scale1[sbase + n + 1]; }
    for (int r = m_row0; r < r1; ++r) {
      const int64_t orow = static_cast<int64_t>(grp.out_row0) + r;
      const float rs = a_row_scale(p, grp, r);
      float g[2] = {0.f, 0.f}, u[2] = {0.f, 0.f};
      for (int s = 0; s < ks; ++s) {
        const float* src = p.partial + s * slice + orow * p.pcols;
        const float2 a = __ldcg(reinterpret_cast<const float2*>(src + n));
        const float2 b = __ldcg(reinterpret_cast<const float2*>(src + N + n));
        g[0] += a.x; g[1] += a.y; u[0] += b.x; u[1] += b.y;
      }
      float o[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float gv = g[j] * rs;
        if (p.scale0 != nullptr) gv *= c0[j];
        float uv = u[j] * rs;
        if (p.scale1 != nullptr) uv *= c1[j];
        o[j] = gv / (1.0f + __expf(-gv)) * uv;
      }
      if (p.out_f32)
        *reinterpret_cast<float2*>(static_cast<float*>(p.out) + orow * N + n) = make_float2(o[0], o[1]);
      else
        *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(p.out) + orow * N + n) = pack_bf16x2(o[0], o[1]);
    }
    return;
  }
  const int n = n_tile * p.bn_out + half * 128 + 4 * lane;
  if (n >= N) return;  // n is a multiple of 4 and N of 8: n + 3 < N
  float cs[4] = {1.f, 1.f, 1.f, 1.f}, cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (p.scale0 != nullptr) cs[j] = p.scale0[sbase + n + j];
    if (EPI == EPI_GELU_BIAS || EPI == EPI_BIAS) cb[j] = p.bias[sbase + n + j];
  }
  for (int r = m_row0; r < r1; ++r) {
    const int64_t orow = static_cast<int64_t>(grp.out_row0) + r;
    const float rs = a_row_scale(p, grp, r);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < ks; ++s) {
      const float4 a = __ldcg(reinterpret_cast<const float4*>(p.partial + s * slice + orow * p.pcols + n));
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
    }
    float o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float z = v[j] * rs;
      if (p.scale0 != nullptr) z *= cs[j];
      if (EPI == EPI_GELU_BIAS || EPI == EPI_BIAS) z += cb[j];
      if (EPI == EPI_GELU_BIAS) z = 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
      o[j] = z;
    }
    if (p.out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * N + n) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
      const uint2 packed = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + orow * N + n) = packed;
    }
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
