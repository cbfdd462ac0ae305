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
// With E4M3 weights the same kernel runs on 8-bit operands: a stage still
// holds 128-byte rows, now 128 K elements, and the MMA kind is f8f6f4 (K = 32
// per instruction); the epilogue multiplies each accumulator row by its
// activation row scale and each column by the weight channel scale.  The A
// rows are E4M3 codes of the activations: one code per element (W8A8), or,
// for bf16 activations, two codes per element (x * 2^k = c1 + c2, rows
// [c1 | c2] of 2K codes): a stage then holds both A tiles and the MMA warp
// issues both terms against the same weight tile into one fp32 sum.
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

#include <algorithm>
#include <atomic>

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
// Prefill loads all 128 token rows of A (4 stages of 48 KB).  When no group
// exceeds 128 rows (decode), m-blocks have 64 rows and only the bma <= 64 rows
// the largest group can fill are loaded; the shared memory saved becomes extra
// stages, i.e. more weight bytes in flight.  The MMA still reads 128 A rows,
// the rows past bma being the start of the next tile in shared memory, and
// their accumulator rows are never stored (with two-term codes the second
// term's rows sit at A rows 64.. and share the MMA).
constexpr int MAX_STAGES = 8;
constexpr int B_HALF = 128 * BK_BYTES;        // 16 KB
constexpr int B_TILE = 2 * B_HALF;            // 32 KB
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, each draining half of a tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
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

template <int EPI, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                           const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                           const __grid_constant__ CUtensorMap tmOut, TcParams p, int bma, int STAGES) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int BK = bk_elems<F8>();
  const int A_TERM = bma * BK_BYTES;              // one A tile (rows x 128 bytes of K)
  const int A_TERMS = F8 ? p.a_terms : 1;         // two-term E4M3 activations: two A tiles per stage
  const int A_TILE = A_TERM * A_TERMS;
  // Stage layout.  Usually [A term 1][A term 2][B].  Packed two-term A (groups
  // of at most 64 rows): [B][A term 1 at rows 0..][A term 2 at rows 64..], so
  // one M=128 MMA multiplies both terms (accumulator lanes 0..63 and 64..127;
  // the 128-row read runs past the stage's end into garbage rows that are
  // never stored).
  const bool PACK = F8 && p.a_pack;
  const int B_OFF = PACK ? 0 : A_TILE;
  const int A_OFF = PACK ? B_TILE : 0;
  const int A2_OFF = PACK ? B_TILE + 64 * BK_BYTES : A_TERM;
  const int STAGE_BYTES = PACK ? B_TILE + 64 * BK_BYTES + A_TERM : A_TILE + B_TILE;
  const int BMX = p.bm;  // rows of an m-block: 128, or 64 for groups of at most 128 rows (decode)
  uint8_t* ctl = ring + STAGES * STAGE_BYTES;
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
        mbar_init(&s.full[i], 1);
        mbar_init(&s.empty[i], 1);
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
          tiles = ((ge.rows + BMX - 1) / BMX) * p.n_tiles;
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
  // packed two-term A: the second term's accumulator rows are one more set of
  // K slices, so every unit writes partial sums and the finalize adds 2 ks slices
  const int ks = choose_ksplit(tiles, gridDim.x, nk, PACK ? p.max_ksplit / 2 : p.max_ksplit);
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.ksplit_out != nullptr) *p.ksplit_out = PACK ? 2 * ks : ks;
  const int total = tiles * ks;  // work units
  volatile int* abort_flag = &s.abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok && !p.test_stall; u += gridDim.x) {
        const UnitInfo ui = decode_unit(s, p, u, ks, nk, BMX);
        const TileInfo& ti = ui.ti;
        const int a_row = (p.a_rows_from_out ? ti.grp.out_row0 : ti.grp.a_row0) + ti.m_idx * BMX;
        const CUtensorMap* mA = (ti.grp.expert == p.shared_slab) ? &tmA2 : &tmA;
        const int b_row = ti.grp.expert * p.n_per_slab + ti.n_idx * p.bn_out;
        for (int kb = ui.kb0; kb < ui.kb1; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&s.full[stage], A_TILE + B_TILE);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          uint8_t* st = ring + stage * STAGE_BYTES;
          uint8_t* sb = st + B_OFF;
          tma_load_2d(st + A_OFF, mA, kb * BK, a_row, &s.full[stage]);
          if (F8 && A_TERMS == 2) tma_load_2d(st + A2_OFF, mA, p.K + kb * BK, a_row, &s.full[stage]);
          if (EPI == EPI_SWIGLU) {
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
          const uint32_t st_base = smem_u32(ring + stage * STAGE_BYTES);
          const uint32_t a_base = st_base + A_OFF;
          const uint32_t b_base = st_base + B_OFF;
          if (F8) {
            // one or two A terms against the same weight tile, one fp32 sum
            // (packed: one MMA covers both terms' rows)
            for (int t = 0; t < (PACK ? 1 : A_TERMS); ++t) {
#pragma unroll
              for (int kk = 0; kk < BK_BYTES / 32; ++kk)  // 32 E4M3 of K per MMA
                tc_mma_f8(d_tmem, smem_desc_sw128(a_base + t * A_TERM + kk * 32), smem_desc_sw128(b_base + kk * 32),
                          kIdescE4m3, (kb > kb0 || kk > 0 || t > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < BK_BYTES / 32; ++kk)  // 16 bf16 of K per MMA
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
  } else {
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;      // which half of the tile's columns it drains
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      const UnitInfo ui = decode_unit(s, p, u, ks, nk, BMX);
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
      // packed two-term A: lane quarters 2, 3 hold the second term's sums of
      // the rows of quarters 0, 1, written as K slices ks .. 2 ks - 1; with
      // 64-row m-blocks and one term, quarters 2, 3 hold no rows of the block
      const int qrow = PACK ? (q & 1) : q;
      if (qrow * 32 < BMX) {  // warp-uniform
        const int row = ti.m_idx * BMX + qrow * 32 + lane;
        const bool valid = row < ti.grp.rows;
        const uint32_t tbase = tmem + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);
        if (PACK)
          epilogue_partial<EPI>(p, ti, tbase, row, valid, ui.split + (q >> 1) * ks, half);
        else if (ks > 1)
          epilogue_partial<EPI>(p, ti, tbase, row, valid, ui.split, half);
        else
          epilogue_store<EPI>(p, ti, tbase, row, valid, lane, half, &tmOut, epi_smem + (warp - 2) * kEpiWarpBytes);
      }
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

template <int EPI, bool F8>
cudaError_t launch_epi(const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB0, const CUtensorMap& mB1,
                       const CUtensorMap& mOut, const TcParams& p, int grid, int bma, int stages, size_t smem,
                       int64_t max_group_rows, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_set{0};  // one bit per device ordinal (host threads may launch concurrently)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set.load(std::memory_order_relaxed) & (1ull << dev))) {
    e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemLimitTc));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set.fetch_or(1ull << dev, std::memory_order_relaxed);
  }
  // programmatic dependent launch: the prologue may overlap the previous kernel
  e = launch_pdl(grouped_gemm_tc_kernel<EPI, F8>, dim3(grid), dim3(kThreads), smem, stream, mA,
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
  // m-blocks of 128 rows; when no group exceeds 128 rows (decode), m-blocks of 64 rows, of which
  // only the rows the largest group can fill (rounded up to 16) are loaded: the shared memory saved
  // becomes extra stages, i.e. more weight bytes in flight
  const bool half = a.max_group_rows > 0 && a.max_group_rows <= 128;
  const int bm = half ? 64 : BM;
  const int bma = half ? static_cast<int>(std::min<int64_t>(64, (a.max_group_rows + 15) & ~int64_t(15))) : BM;
  const int terms = a.fp8 && a.a_terms == 2 ? 2 : 1;  // two-term E4M3 activations: A rows of 2K codes
  // both terms in one MMA (64-row m-blocks; the split-K buffer holds the second term's sums)
  const bool pack = terms == 2 && half && p.max_ksplit >= 2;
  const size_t stage_bytes = pack ? static_cast<size_t>(B_TILE + 64 * BK_BYTES + bma * BK_BYTES)
                                  : static_cast<size_t>(bma) * BK_BYTES * terms + B_TILE;
  const int eb = a.fp8 ? 1 : 2;  // element bytes of A and B
  int stages = static_cast<int>((kSmemLimitTc - kCtlBytes) / stage_bytes);
  if (stages > MAX_STAGES) stages = MAX_STAGES;
  const size_t smem = stages * stage_bytes + kCtlBytes;
  CUtensorMap mA, mA2, mB0, mB1, mOut;
  // bf16 outputs: full 32-row quarters go out as bulk tensor stores; fp32 outputs store row by row
  TcParams pp = p;
  pp.tma_out = !a.out_f32 && make_store_map(&mOut, a.out, a.out_rows, a.N, 2) ? 1 : 0;
  if (!pp.tma_out) memset(&mOut, 0, sizeof(mOut));
  pp.a_terms = terms;
  pp.a_pack = pack ? 1 : 0;
  pp.bm = bm;
  if (!make_map(&mA, a.a, a.a_rows, a.K * terms, bma, eb)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    if (!make_map(&mA2, a.a_shared, a.a_shared_rows, a.K * terms, bma, eb)) return cudaErrorInvalidValue;
  } else {
    mA2 = mA;
  }
  if (!make_map(&mB0, a.b0, a.b_rows, a.K, 128, eb)) return cudaErrorInvalidValue;
  if (a.epilogue == EPI_SWIGLU) {
    if (!make_map(&mB1, a.b1, a.b_rows, a.K, 128, eb)) return cudaErrorInvalidValue;
  } else {
    mB1 = mB0;
  }
  // upper bound of the tile count: every group may add one partial m-block
  const int64_t bound = (a.max_total_rows / bm + a.num_groups) * static_cast<int64_t>(p.n_tiles);
  const int grid = static_cast<int>(bound < num_sms ? (bound > 0 ? bound : 1) : num_sms);
  if (a.fp8) {  // E4M3 x E4M3 runs SwiGLU experts only
    switch (a.epilogue) {
      case EPI_SWIGLU:
        return launch_epi<EPI_SWIGLU, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
      case EPI_NONE:
        return launch_epi<EPI_NONE, true>(mA, mA2, mB0, mB1, mOut, pp, grid, bma, stages, smem, a.max_group_rows, stream);
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
