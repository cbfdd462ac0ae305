// Grouped expert GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// jsqmd.com "第11章 MoE模型推理" 11.1.2: the B*L*K expert forwards of a layer
// are grouped by expert and run together; plumephp.com "MoE 混合专家推理",
// activation-memory block ("sequence expert"): feed all of an expert's tokens
// to it as one large GEMM.  Here every expert group is a slice of rows of one
// A buffer, and one persistent launch runs all groups:
//
//   out[out_row0 + r, n] = epi( sum_k A[a_row0 + r, k] * W[expert][n, k] )
//
// Up projection, SwiGLU: W = [W_gate rows n0..n0+127 ; W_up rows n0..n0+127]
// forms one 256-row B tile, so one M=128 x N=256 MMA produces the gate and the
// up accumulators side by side in TMEM and the epilogue writes
// silu(gate) * up (x per-channel scales for FP8 weights) as bf16.
// Down projection: 256 output columns per tile, optional bias / scale.
//
// With E4M3 activations and weights (W8A8) the same kernel runs on 8-bit
// operands: a stage still holds 128-byte rows, now 128 K elements, and the
// MMA kind is f8f6f4 (K = 32 per instruction); the epilogue multiplies each
// accumulator row by its activation row scale and each column by the weight
// channel scale.
//
// Structure (one CTA per SM, 320 threads):
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 (bf16, 128-byte
//               swizzle) per stage into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (kind::f16, fp32 accumulate) and tcgen05.commit;
//   warps 2-9   epilogue, two warps per 32-lane TMEM quarter, each draining
//               half of the tile's columns: tcgen05.ld, activation, then a
//               bulk tensor store per 32 x 32 box (or row stores for a group's
//               last, partial quarter).
// Two 256-column accumulators let the epilogue of tile i overlap the MMAs of
// tile i+1.  The tile list (group, n-block, m-block; m fastest, so the CTAs
// in flight share weight tiles through L2) is derived on the device from the
// group table: no host synchronisation on routing results.
//
// Every mbarrier wait is bounded in time; a CTA that gives up raises a flag
// in shared memory and the status block, waits for its own copies and MMAs
// in flight, frees its TMEM and exits.  No load uses cluster multicast.
#include <math.h>

#include <stdlib.h>
#include <string.h>

#include "gemm_common.cuh"
#include "pdl.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int BM = 128;
constexpr int BK_BYTES = 128;  // one swizzle row: 64 bf16 or 128 E4M3 elements of K per stage
// Ring: one stage = A rows (bma x 64 bf16, bma <= 128) then B (256 x 64 bf16).
// Prefill loads all 128 token rows of A (4 stages of 48 KB).  When every group
// fits in bma < 128 rows (decode), only those rows are loaded and the shared
// memory saved becomes extra stages, i.e. more weight bytes in flight; the
// MMA still reads 128 A rows, the rows past bma being the start of the same
// stage's B tile, and their accumulator rows are never stored.
constexpr int MAX_STAGES = 8;
constexpr int B_HALF = 128 * BK_BYTES;        // 16 KB
constexpr int B_TILE = 2 * B_HALF;            // 32 KB
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, each draining half of a tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
// E4M3 weights with bf16 activations (W8): eight more warps decode each landed
// E4M3 weight tile into the bf16 B tile of its stage.
constexpr int kConvWarps = 8;
constexpr int kConvGroups = 2;  // the two K steps of a landing buffer are decoded side by side
constexpr int kGroupThreads = 32 * kConvWarps / kConvGroups;
constexpr int kThreadsW8 = kThreads + 32 * kConvWarps;
constexpr int kMaxLandStages = 8;          // landing buffers of E4M3 weight tiles (at most)
constexpr int LAND_BYTES = 256 * 128;      // 256 weight rows x 128 E4M3 codes (two bf16 K steps)
constexpr uint32_t kIdescBf16 = idesc_bf16_f32(128, 256);
constexpr uint32_t kIdescE4m3 = idesc_e4m3_f32(128, 256);

// K elements per stage of the bf16 (F8 = false) and E4M3 (F8 = true) kernels
template <bool F8>
constexpr int bk_elems() {
  return F8 ? BK_BYTES : BK_BYTES / 2;
}

struct SmemCtl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t lfull[kMaxLandStages];  // W8: an E4M3 weight tile has landed
  uint64_t ldone[kMaxLandStages];  // W8: the first K step of a two-step landing buffer is decoded
  int land_parity[kMaxLandStages]; // W8: parity of the latest copy into each landing buffer (-1: none)
  int conv_ok[kConvGroups];        // W8: each converter group's shared go / give-up decision
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int ksplit;
  int tile_start[kMaxGroups + 1];
};

constexpr size_t kSmemLimitTc = 232448;  // 227 KB per CTA
// epilogue staging: one 32 x 32 box (fp32 at most) per epilogue warp, 128-byte aligned
constexpr int kEpiWarpBytes = 32 * 32 * 2;  // bf16 boxes (fp32 outputs store row by row)
constexpr size_t kCtlBytes = sizeof(SmemCtl) + 1024 + 128 + kEpiWarps * kEpiWarpBytes;  // control, staging, slack

__device__ __forceinline__ bool wait_timed(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never);
}

struct TileInfo {
  GroupEntry grp;
  int m_idx, n_idx;
};

__device__ __forceinline__ TileInfo decode_tile(const SmemCtl& s, const TcParams& p, int tt, int bm = BM) {
  int lo = 0, hi = p.num_groups;  // find g: tile_start[g] <= tt < tile_start[g+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= tt)
      lo = mid;
    else
      hi = mid;
  }
  TileInfo ti;
  ti.grp = group_at(p, lo);
  const int mt = (ti.grp.rows + bm - 1) / bm;
  const int local = tt - s.tile_start[lo];
  ti.n_idx = local / mt;
  ti.m_idx = local - ti.n_idx * mt;
  return ti;
}

struct UnitInfo {
  TileInfo ti;
  int split, kb0, kb1;
};

__device__ __forceinline__ UnitInfo decode_unit(const SmemCtl& s, const TcParams& p, int u, int ks, int nk,
                                                int bm = BM) {
  UnitInfo ui;
  const int tt = u / ks;
  ui.split = u - tt * ks;
  ui.ti = decode_tile(s, p, tt, bm);
  ui.kb0 = static_cast<int>((static_cast<int64_t>(ui.split) * nk) / ks);
  ui.kb1 = static_cast<int>((static_cast<int64_t>(ui.split + 1) * nk) / ks);
  return ui;
}

// Epilogue of one 32-row quarter of a tile: thread `lane` owns accumulator
// row `row` (and its activation row scale rs).  The per-column operands
// (weight-channel scales, biases) are loaded once per 32-column chunk, lane j
// holding column n + j, and handed to every lane by shuffles; SiLU uses the
// fast reciprocal-based division.
//
// A warp whose 32 rows all belong to the group (every quarter but a group's
// last) writes each 32-column chunk into its shared-memory box and stores it
// with one bulk tensor store (full 128-byte lines instead of 32 scattered
// 16-byte pieces per store instruction); a partial quarter stores row by row.
template <int EPI>
__device__ __forceinline__ void epilogue_store(const TcParams& p, const TileInfo& ti, uint32_t tbase, int row,
                                               bool valid, int lane, int half, const CUtensorMap* tm_out,
                                               uint8_t* ebuf) {
  const int N = p.N;
  const int64_t orow = static_cast<int64_t>(ti.grp.out_row0) + row;
  const bool full = p.tma_out && (row - lane) + 32 <= ti.grp.rows;  // warp-uniform
  const int64_t sbase = static_cast<int64_t>(ti.grp.expert) * N;
  const float rs = valid ? a_row_scale(p, ti.grp, row) : 1.0f;
  constexpr int kChunks = (EPI == EPI_SWIGLU) ? 4 : 8;
  constexpr bool kBias = EPI == EPI_GELU_BIAS || EPI == EPI_BIAS;
  for (int c = half * (kChunks / 2); c < (half + 1) * (kChunks / 2); ++c) {
    const int n = ti.n_idx * p.bn_out + c * 32;
    const bool col_ok = n + lane < N;
    float cs0 = 1.0f, cs1 = 1.0f, cb = 0.0f;  // this lane's column: channel scales, bias
    if (col_ok) {
      if (p.scale0 != nullptr) cs0 = __ldg(p.scale0 + sbase + n + lane);
      if (EPI == EPI_SWIGLU && p.scale1 != nullptr) cs1 = __ldg(p.scale1 + sbase + n + lane);
      if (kBias) cb = __ldg(p.bias + sbase + n + lane);
    }
    uint32_t r0[32];
    float v[32];
    if (EPI == EPI_SWIGLU) {
      uint32_t r1[32];
      tmem_ld_32x32b_x32(tbase + c * 32, r0);
      tmem_ld_32x32b_x32(tbase + 128 + c * 32, r1);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float g = __uint_as_float(r0[j]) * rs * __shfl_sync(0xFFFFFFFFu, cs0, j);
        const float u = __uint_as_float(r1[j]) * rs * __shfl_sync(0xFFFFFFFFu, cs1, j);
        v[j] = __fdividef(g, 1.0f + __expf(-g)) * u;
      }
    } else {
      tmem_ld_32x32b_x32(tbase + c * 32, r0);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float z = __uint_as_float(r0[j]) * rs * __shfl_sync(0xFFFFFFFFu, cs0, j);
        if (kBias) z += __shfl_sync(0xFFFFFFFFu, cb, j);
        if (EPI == EPI_GELU_BIAS) z = 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
        v[j] = z;
      }
    }
    if (full) {
      if (lane == 0) bulk_wait_read_all();  // the previous box has been read out
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j) stg16(ebuf + lane * 64 + 16 * j, pack16<__nv_bfloat16>(v + 8 * j));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && n < N) {
        tma_store_2d(tm_out, ebuf, n, static_cast<int>(orow - lane));
        bulk_commit();
      }
      continue;
    }
    if (!valid) continue;
    if (p.out_f32) {
      float* o = static_cast<float*>(p.out) + orow * N + n;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (n + 4 * j + 4 <= N) stg16(o + 4 * j, pack16<float>(v + 4 * j));
    } else {
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + orow * N + n;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (n + 8 * j + 8 <= N) stg16(o + 8 * j, pack16<__nv_bfloat16>(v + 8 * j));
    }
  }
}

// Split-K epilogue: raw fp32 accumulators of this unit's K range go to its
// slice of the partial buffer, for the warp's region of the tile: rows of its
// TMEM lane quarter, and half of the tile's columns -- SwiGLU: output columns
// half*64 .. +63, i.e. gate chunks {2 half, 2 half + 1} and up chunks
// {4 + 2 half, 5 + 2 half}, gate stored at column n and up at N + n; other
// epilogues: columns half*128 .. +127.
template <int EPI>
__device__ __forceinline__ void epilogue_partial(const TcParams& p, const TileInfo& ti, uint32_t tbase, int row,
                                                 bool valid, int split, int half) {
  const int N = p.N;
  const int64_t orow = static_cast<int64_t>(ti.grp.out_row0) + row;
  float* base = p.partial + (static_cast<int64_t>(split) * p.out_rows + orow) * p.pcols;
  for (int i = 0; i < 4; ++i) {
    const int c = (EPI == EPI_SWIGLU) ? ((i < 2 ? 0 : 4) + 2 * half + (i & 1)) : (half * 4 + i);
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c * 32, r);
    tmem_ld_wait();
    if (!valid) continue;
    int n, col;
    if (EPI == EPI_SWIGLU) {
      n = ti.n_idx * p.bn_out + (c & 3) * 32;
      col = (c < 4 ? 0 : N) + n;
    } else {
      n = ti.n_idx * p.bn_out + c * 32;
      col = n;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (n + 4 * j + 4 <= N)
        stg16(base + col + 4 * j, make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]));
    }
  }
}

// Four E4M3 codes (bytes of w, lowest first) -> four bf16 values (lo: codes
// 0, 1; hi: codes 2, 3), exactly: E4M3 -> f16 is exact (every E4M3 value,
// subnormals included, is a normal f16 or zero), f16 -> f32 is exact, and the
// f32 -> bf16 rounding keeps the value (at most four significant bits, inside
// bf16's exponent range).  The f16 -> bf16 step goes through f32 because the
// packed f32 -> bf16x2 conversion is one instruction for two values.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c0, c1, a, b, c, d;\n\t.reg .b32 h0, h1;\n\t.reg .f32 fa, fb, fc, fd;\n\t"
      "mov.b32 {c0, c1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 h0, c0;\n\t"
      "cvt.rn.f16x2.e4m3x2 h1, c1;\n\t"
      "mov.b32 {a, b}, h0;\n\t"
      "cvt.f32.f16 fa, a;\n\t"
      "cvt.f32.f16 fb, b;\n\t"
      "cvt.rn.bf16x2.f32 %0, fb, fa;\n\t"
      "mov.b32 {c, d}, h1;\n\t"
      "cvt.f32.f16 fc, c;\n\t"
      "cvt.f32.f16 fd, d;\n\t"
      "cvt.rn.bf16x2.f32 %1, fd, fc;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// W8: one converter group (kGroupThreads threads) decodes the 64 codes of
// one K step from each of the 256 rows of a landing buffer (rows of 128
// bytes, two K steps; `land` points at the step's first code of row 0) into
// the stage's 256 x 128-byte bf16 B tile in the 128-byte swizzled layout the
// MMA reads (16-byte chunk j of row r at chunk j ^ (r & 7)).  Thread gt takes
// the 16-code pieces gt + kGroupThreads i.
__device__ __forceinline__ void convert_tile_w8(const uint8_t* land, uint8_t* b16, int gt) {
#pragma unroll 2
  for (int i = 0; i < 1024 / kGroupThreads; ++i) {
    const int piece = gt + kGroupThreads * i;  // 1024 pieces of 16 codes
    const int r = piece >> 2, q4 = piece & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(land + r * 128 + q4 * 16);
    uint32_t o[8];
    e4m3x4_to_bf16x4(v.x, o[0], o[1]);
    e4m3x4_to_bf16x4(v.y, o[2], o[3]);
    e4m3x4_to_bf16x4(v.z, o[4], o[5]);
    e4m3x4_to_bf16x4(v.w, o[6], o[7]);
    uint8_t* row = b16 + r * BK_BYTES;
    const int sw = r & 7;
    *reinterpret_cast<uint4*>(row + (((2 * q4) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(row + (((2 * q4 + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int EPI, bool F8, bool W8>
__global__ void __launch_bounds__(W8 ? kThreadsW8 : kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                           const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                           const __grid_constant__ CUtensorMap tmOut, TcParams p, int bma, int STAGES) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int BK = bk_elems<F8>();
  const int A_TILE = bma * BK_BYTES;
  const int STAGE_BYTES = A_TILE + B_TILE;
  uint8_t* land = ring + STAGES * STAGE_BYTES;  // W8 landing buffers (1024-byte aligned)
  const int LAND = W8 ? p.land_stages : 0;       // W8 landing buffers in use
  uint8_t* ctl = land + LAND * LAND_BYTES;
  SmemCtl& s = *reinterpret_cast<SmemCtl*>(ctl);
  uint8_t* epi_smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(ctl + sizeof(SmemCtl)) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = lane_id();

  // Prologue that needs nothing from earlier kernels (barriers, TMEM, tensor
  // map prefetch) runs first; under programmatic dependent launch it overlaps
  // the previous kernel, and the wait below is where this grid first needs
  // that kernel's results (group table, A rows, partial buffer).
  if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        mbar_init(&s.full[i], W8 ? 2 : 1);  // W8: the A copy's arrival plus the converters'
        mbar_init(&s.empty[i], 1);
      }
      if (W8)
        for (int i = 0; i < LAND; ++i) {
          mbar_init(&s.lfull[i], 1);
          mbar_init(&s.ldone[i], 1);
          s.land_parity[i] = -1;
        }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&s.tfull[i], 1);
        mbar_init(&s.tempty[i], 32 * kEpiWarps);
      }
      mbar_init(&s.drain, 1);
      s.abort = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  } else if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  pdl_wait();
  pdl_trigger();
  // per-group tile counts -> exclusive prefix (warp 0)
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.num_groups; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < p.num_groups) {
        const GroupEntry ge = group_at(p, g);
        if (group_ok(ge, p))
          tiles = ((ge.rows + BM - 1) / BM) * p.n_tiles;
        else if (ge.rows != 0)
          report(p.status, MOE_STATUS_BAD_GROUP, -1);
      }
      int incl = tiles;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < p.num_groups) s.tile_start[g] = carry + incl - tiles;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) s.tile_start[p.num_groups] = carry;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = s.tmem_base;
  const int nk = (p.K + BK - 1) / BK;
  const int tiles = s.tile_start[p.num_groups];
  const int ks = choose_ksplit(tiles, gridDim.x, nk, p.max_ksplit);
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.ksplit_out != nullptr) *p.ksplit_out = ks;
  const int total = tiles * ks;  // work units
  volatile int* abort_flag = &s.abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok && !p.test_stall; u += gridDim.x) {
        const UnitInfo ui = decode_unit(s, p, u, ks, nk);
        const TileInfo& ti = ui.ti;
        const int a_row = (p.a_rows_from_out ? ti.grp.out_row0 : ti.grp.a_row0) + ti.m_idx * BM;
        const CUtensorMap* mA = (ti.grp.expert == p.shared_slab) ? &tmA2 : &tmA;
        const int b_row = ti.grp.expert * p.n_per_slab + ti.n_idx * p.bn_out;
        for (int kb = ui.kb0; kb < ui.kb1; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&s.full[stage], W8 ? A_TILE : STAGE_BYTES);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          uint8_t* sa = ring + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_TILE;
          tma_load_2d(sa, mA, kb * BK, a_row, &s.full[stage]);
          if (W8) {
            // the converters fill this stage's B tile
          } else if (EPI == EPI_SWIGLU) {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &s.full[stage]);
            tma_load_2d(sb + B_HALF, &tmB1, kb * BK, b_row, &s.full[stage]);
          } else {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &s.full[stage]);
            tma_load_2d(sb + B_HALF, &tmB0, kb * BK, b_row + 128, &s.full[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
        // let the copies already issued land before the CTA exits
        for (int i = 0; i < STAGES; ++i)
          if (armed & (1u << i)) wait_timed(&s.full[i], (armed_phase >> i) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++local) {
        const int split = u % ks;
        const int kb0 = static_cast<int>((static_cast<int64_t>(split) * nk) / ks);
        const int kb1 = static_cast<int>((static_cast<int64_t>(split + 1) * nk) / ks);
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * ACC_COLS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + stage * STAGE_BYTES);
          const uint32_t b_base = a_base + A_TILE;
#pragma unroll
          for (int kk = 0; kk < BK_BYTES / 32; ++kk) {  // 32 bytes of K per MMA (16 bf16 or 32 E4M3)
            if (F8)
              tc_mma_f8(d_tmem, smem_desc_sw128(a_base + kk * 32), smem_desc_sw128(b_base + kk * 32), kIdescE4m3,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
            else
              tc_mma_f16(d_tmem, smem_desc_sw128(a_base + kk * 32), smem_desc_sw128(b_base + kk * 32), kIdescBf16,
                         (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&s.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&s.tfull[acc]);
      }
      // every MMA this thread issued must finish before TMEM is released
      tc_commit(&s.drain);
      wait_timed(&s.drain, 0);
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
      }
    }
    __syncwarp();
  } else if (W8 && warp >= 2 + kEpiWarps) {
    // W8 converters, two groups of four warps.  A landing buffer holds the
    // E4M3 codes of two K steps of a weight tile (256 rows x 128 bytes: DRAM
    // reads of 128 contiguous bytes per row); group 0 decodes the first K
    // step, group 1 the second, side by side.  For its K step a group waits
    // for the codes to land and for the stage's B tile to be free, decodes,
    // then lets the MMA go (second arrival on the stage's full barrier).  The
    // group decoding a buffer's last K step refills it with the pair LAND
    // pairs ahead (group 1 first waits for group 0's half: ldone).  Both
    // groups walk the whole K-step sequence, so they agree on stages, phases
    // and buffers.  Each group's first thread waits on the barriers; the go /
    // give-up decision reaches the group through shared memory.
    const int ct = threadIdx.x - (2 + kEpiWarps) * 32;
    const int g = ct / kGroupThreads, gt = ct % kGroupThreads;
    // the sequence of K-step pairs, walked twice: `cur` for decoding, `ahd` for issuing copies
    struct Seq {
      int u, kb, kb1;  // unit, first K step of the pair, end of the unit's K range
    };
    auto seq_begin = [&](Seq& q) {
      q.u = blockIdx.x;
      q.kb = 0;
      q.kb1 = 0;
      while (q.u < total) {
        const UnitInfo ui = decode_unit(s, p, q.u, ks, nk);
        q.kb = ui.kb0;
        q.kb1 = ui.kb1;
        if (q.kb < q.kb1) return;
        q.u += gridDim.x;
      }
    };
    auto seq_next = [&](Seq& q) {
      q.kb += 2;
      if (q.kb < q.kb1) return;
      q.u += gridDim.x;
      while (q.u < total) {
        const UnitInfo ui = decode_unit(s, p, q.u, ks, nk);
        q.kb = ui.kb0;
        q.kb1 = ui.kb1;
        if (q.kb < q.kb1) return;
        q.u += gridDim.x;
      }
    };
    auto issue = [&](const Seq& q, int l, uint32_t parity) {  // E4M3 codes of pair q into landing buffer l
      const UnitInfo ui = decode_unit(s, p, q.u, ks, nk);
      const int b_row = ui.ti.grp.expert * p.n_per_slab + ui.ti.n_idx * p.bn_out;
      uint8_t* dst = land + l * LAND_BYTES;
      s.land_parity[l] = static_cast<int>(parity);
      mbar_arrive_expect_tx(&s.lfull[l], LAND_BYTES);
      if (EPI == EPI_SWIGLU) {
        tma_load_2d(dst, &tmB0, q.kb * BK, b_row, &s.lfull[l]);
        tma_load_2d(dst + LAND_BYTES / 2, &tmB1, q.kb * BK, b_row, &s.lfull[l]);
      } else {
        tma_load_2d(dst, &tmB0, q.kb * BK, b_row, &s.lfull[l]);
        tma_load_2d(dst + LAND_BYTES / 2, &tmB0, q.kb * BK, b_row + 128, &s.lfull[l]);
      }
    };
    Seq cur, ahd;
    seq_begin(cur);
    seq_begin(ahd);
    if (g == 0 && gt == 0 && !p.test_stall) {
      for (int l = 0; l < LAND && ahd.u < total; ++l) {
        issue(ahd, l, 0u);
        seq_next(ahd);
      }
    } else {
      for (int l = 0; l < LAND && ahd.u < total; ++l) seq_next(ahd);
    }
    int stage = 0, l = 0;
    uint32_t phase = 0, lphase = 0, ld_bits = 0;
    bool ok = true;
    while (cur.u < total && ok) {
      const int n = min(2, cur.kb1 - cur.kb);  // K steps in this pair
      for (int h = 0; h < n; ++h) {
        if (h == g) {
          if (gt == 0) {
            const int go = !p.test_stall && mbar_wait(&s.lfull[l], lphase, abort_flag) &&
                           mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag);
            s.conv_ok[g] = go;
          }
          named_bar_sync(1 + g, kGroupThreads);
          if (!s.conv_ok[g]) {
            ok = false;
            break;
          }
          convert_tile_w8(land + l * LAND_BYTES + h * 64, ring + stage * STAGE_BYTES + A_TILE, gt);
          fence_proxy_async_smem();  // generic-proxy writes before the tensor core's reads
          named_bar_sync(1 + g, kGroupThreads);
          if (gt == 0) {
            mbar_arrive(&s.full[stage]);
            if (g == 0 && n == 2) mbar_arrive(&s.ldone[l]);
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      // the group that decoded the pair's last K step refills the buffer
      if (g == n - 1 && gt == 0 && ahd.u < total) {
        if (n == 2 && !mbar_wait(&s.ldone[l], (ld_bits >> l) & 1u, abort_flag)) {
          ok = false;
        } else {
          issue(ahd, l, (lphase + 1u) & 1u);
        }
      }
      if (n == 2) ld_bits ^= 1u << l;
      if (g == n - 1 && gt == 0) s.conv_ok[g] = ok;
      named_bar_sync(1 + g, kGroupThreads);
      if (g == n - 1 && !s.conv_ok[g]) ok = false;
      if (!ok) break;
      seq_next(ahd);
      seq_next(cur);
      if (++l == LAND) {
        l = 0;
        lphase ^= 1u;
      }
    }
    if (!ok && gt == 0) {
      *abort_flag = 1;
      report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
      // let the copies already issued land before the CTA exits
      for (int i = 0; i < LAND; ++i)
        if (s.land_parity[i] >= 0) wait_timed(&s.lfull[i], static_cast<uint32_t>(s.land_parity[i]));
    }
  } else {
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;      // which half of the tile's columns it drains
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      const UnitInfo ui = decode_unit(s, p, u, ks, nk);
      const TileInfo& ti = ui.ti;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(&s.tfull[acc], acc_phase, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
        }
        break;
      }
      tc_fence_after();
      const int row = ti.m_idx * BM + q * 32 + lane;
      const bool valid = row < ti.grp.rows;
      const uint32_t tbase = tmem + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);
      if (ks > 1)
        epilogue_partial<EPI>(p, ti, tbase, row, valid, ui.split, half);
      else
        epilogue_store<EPI>(p, ti, tbase, row, valid, lane, half, &tmOut, epi_smem + (warp - 2) * kEpiWarpBytes);
      tc_fence_before();
      mbar_arrive(&s.tempty[acc]);
    }
  }

  if (warp >= 2 && warp < 2 + kEpiWarps && lane == 0) bulk_wait_all();  // this warp's output boxes are written
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int EPI, bool F8, bool W8 = false>
cudaError_t launch_epi(const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB0, const CUtensorMap& mB1,
                       const CUtensorMap& mOut, const TcParams& p, int grid, int bma, int stages, size_t smem,
                       int64_t max_group_rows, cudaStream_t stream) {
  static uint64_t attr_set = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<EPI, F8, W8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemLimitTc));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  // programmatic dependent launch: the prologue may overlap the previous kernel
  e = launch_pdl(grouped_gemm_tc_kernel<EPI, F8, W8>, dim3(grid), dim3(W8 ? kThreadsW8 : kThreads), smem, stream, mA,
                 mA2, mB0, mB1, mOut, p, bma, stages);
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess || p.max_ksplit <= 1) return e;
  dim3 fgrid((p.N + 1023) / 1024, static_cast<unsigned>(max_group_rows), p.num_groups);
  e = launch_pdl(splitk_finalize_kernel<EPI>, fgrid, dim3(256), 0, stream, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

// Token-rows kernel launch; `p` is filled by launch_grouped_gemm_tc.
cudaError_t launch_grouped_gemm_single(const GemmArgs& a, const gemm::TcParams& p, int num_sms, cudaStream_t stream) {
  // A rows loaded per stage: all 128, or (every group fitting) the largest group rounded up to 16
  int bma = BM;
  if (a.max_group_rows > 0 && a.max_group_rows <= 64) bma = static_cast<int>((a.max_group_rows + 15) & ~int64_t(15));
  const size_t stage_bytes = static_cast<size_t>(bma) * BK_BYTES + B_TILE;
  const int eb = a.fp8 ? 1 : 2;  // element bytes of A and B
  const bool w8 = a.w8 != 0 && !a.fp8;
  int stages, land = 0;
  if (w8) {
    // E4M3 weights: the HBM latency is covered by the landing buffers (a
    // weight tile is decoded into a bf16 stage only when the MMA is about to
    // need it), so three bf16 stages and as many landing buffers as fit
    stages = 3;
    land = static_cast<int>((kSmemLimitTc - kCtlBytes - stages * stage_bytes) / LAND_BYTES);
    if (land < 2) {
      stages = 2;
      land = static_cast<int>((kSmemLimitTc - kCtlBytes - stages * stage_bytes) / LAND_BYTES);
    }
    if (land > kMaxLandStages) land = kMaxLandStages;
    if (land < 2) return cudaErrorInvalidValue;
  } else {
    stages = static_cast<int>((kSmemLimitTc - kCtlBytes) / stage_bytes);
    if (stages > MAX_STAGES) stages = MAX_STAGES;
  }
  const size_t land_bytes = static_cast<size_t>(land) * LAND_BYTES;
  const size_t smem = stages * stage_bytes + land_bytes + kCtlBytes;
  CUtensorMap mA, mA2, mB0, mB1, mOut;
  // bf16 outputs: full 32-row quarters go out as bulk tensor stores; fp32 outputs store row by row
  TcParams pp = p;
  pp.land_stages = land;
  pp.tma_out = !a.out_f32 && make_store_map(&mOut, a.out, a.out_rows, a.N, 2) ? 1 : 0;
  if (!pp.tma_out) memset(&mOut, 0, sizeof(mOut));
  if (!make_map(&mA, a.a, a.a_rows, a.K, bma, eb)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    if (!make_map(&mA2, a.a_shared, a.a_shared_rows, a.K, bma, eb)) return cudaErrorInvalidValue;
  } else {
    mA2 = mA;
  }
  if (w8) {
    // E4M3 weight tiles of one bf16 K step: 64 codes (64 bytes) x 128 rows, unswizzled
    if (!make_map_w8(&mB0, a.b0, a.b_rows, a.K)) return cudaErrorInvalidValue;
    if (a.epilogue == EPI_SWIGLU) {
      if (!make_map_w8(&mB1, a.b1, a.b_rows, a.K)) return cudaErrorInvalidValue;
    } else {
      mB1 = mB0;
    }
  } else {
    if (!make_map(&mB0, a.b0, a.b_rows, a.K, 128, eb)) return cudaErrorInvalidValue;
    if (a.epilogue == EPI_SWIGLU) {
      if (!make_map(&mB1, a.b1, a.b_rows, a.K, 128, eb)) return cudaErrorInvalidValue;
    } else {
      mB1 = mB0;
    }
  }
  // upper bound of the tile count: every group may add one partial m-block
  const int64_t bound = (a.max_total_rows / BM + a.num_groups) * static_cast<int64_t>(p.n_tiles);
  const int grid = static_cast<int>(bound < num_sms ? (bound > 0 ? bound : 1) : num_sms);
  if (a.fp8) {  // W8A8 runs SwiGLU experts only
    switch (a.epilogue) {
      case EPI_SWIGLU:
        return launch_epi<EPI_SWIGLU, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
      case EPI_NONE:
        return launch_epi<EPI_NONE, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (w8) {  // E4M3 weights, bf16 activations: SwiGLU experts only
    switch (a.epilogue) {
      case EPI_SWIGLU:
        return launch_epi<EPI_SWIGLU, false, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem,
                                                   a.max_group_rows, stream);
      case EPI_NONE:
        return launch_epi<EPI_NONE, false, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem,
                                                 a.max_group_rows, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.epilogue) {
    case EPI_SWIGLU:
      return launch_epi<EPI_SWIGLU, false>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
    case EPI_GELU_BIAS:
      return launch_epi<EPI_GELU_BIAS, false>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
    case EPI_BIAS:
      return launch_epi<EPI_BIAS, false>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
    case EPI_NONE:
      return launch_epi<EPI_NONE, false>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
