// Grouped expert GEMM, one CTA per tile, weights as the M operand (tcgen05).
//
// Same operation as the token-rows kernel (jsqmd.com "第11章 MoE模型推理"
// 11.1.2: the S*K expert forwards run grouped by expert), arranged for small
// and ragged groups:
//
//   D[feature, token] = sum_k W[expert][feature, k] * A[token, k]
//
// A tile is 128 weight rows (M, TMEM lanes) by a block of up to `ntb` tokens
// (N, a multiple of 16, TMEM columns).  `ntb` is chosen per launch from the
// largest group: 256 for prefill, 16 for one-token decode.  The shared-memory
// ring holds 16 KB of weights and ntb*128 bytes of tokens per K-step of 64,
// and as many stages as fit: 4 at ntb=256, 11 at ntb=16, so a decode launch
// keeps ~180 KB of weight bytes in flight per SM instead of 128 KB of useful
// bytes next to 64 KB of padding token rows.  A group's last token block is
// padded by at most 15 rows.
//
// SwiGLU: the 128 weight rows are 64 gate and 64 up rows interleaved in blocks
// of 16, so lanes 0-15 / 16-31 of every TMEM quarter hold gate / up of the
// same 16 features (one shuffle pairs them).  Split-K for small row spaces,
// bounded waits and the roles (warp 0 TMA, warp 1 TMEM + MMA, warps 2-5
// epilogue) are as in the token-rows kernel.  No load uses cluster multicast.
#include "gemm_wt_epilogue.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int WB_K = 64;
constexpr int W_MAX_STAGES = 12;
constexpr int W_W_BYTES = 128 * WB_K * 2;  // weights per stage
constexpr int W_ACC_COLS = 256;
constexpr int W_TMEM_COLS = 512;
constexpr int W_THREADS = 192;
constexpr int W_TBUF = 16 * 32 * 2;  // per epilogue warp

struct WtCtl {
  uint64_t full[W_MAX_STAGES];
  uint64_t empty[W_MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[kMaxGroups + 1];
};
constexpr size_t kWtCtlBytes = (sizeof(WtCtl) + 127) & ~size_t(127);
constexpr size_t kSmemLimit = 232448;  // 227 KB per CTA
constexpr size_t kWtFixed = kWtCtlBytes + 4 * W_TBUF + 1024;  // control, transpose buffers, alignment slack

template <int EPI>
struct WtShape {
  static constexpr int FEAT = EPI == EPI_SWIGLU ? 64 : 128;  // output features per tile
};

struct WtUnit {
  GroupEntry grp;
  int fb, tb, split, kb0, kb1, nt;
};

__device__ __forceinline__ WtUnit wt_unit(const WtCtl& s, const TcParams& p, int u, int ks, int nk, int ntb) {
  WtUnit wu;
  const int tt = u / ks;
  wu.split = u - tt * ks;
  int lo = 0, hi = p.num_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= tt)
      lo = mid;
    else
      hi = mid;
  }
  wu.grp = group_at(p, lo);
  const int nblk = (wu.grp.rows + ntb - 1) / ntb;
  const int local = tt - s.tile_start[lo];
  wu.fb = local / nblk;
  wu.tb = local - wu.fb * nblk;
  wu.nt = min(ntb, wu.grp.rows - wu.tb * ntb);
  wu.kb0 = static_cast<int>((static_cast<int64_t>(wu.split) * nk) / ks);
  wu.kb1 = static_cast<int>((static_cast<int64_t>(wu.split + 1) * nk) / ks);
  return wu;
}

template <int EPI>
__global__ void __launch_bounds__(W_THREADS, 1)
    grouped_gemm_wt_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmT2,
                           const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                           TcParams p, int ntb, int stages) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = W_W_BYTES + ntb * WB_K * 2;
  WtCtl& s = *reinterpret_cast<WtCtl*>(ring + stages * stage_bytes);
  __nv_bfloat16* tbufs = reinterpret_cast<__nv_bfloat16*>(ring + stages * stage_bytes + kWtCtlBytes);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  constexpr int FEAT = WtShape<EPI>::FEAT;
  const int nfb = (p.N + FEAT - 1) / FEAT;

  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.num_groups; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < p.num_groups) {
        const GroupEntry ge = group_at(p, g);
        if (group_ok(ge, p))
          tiles = ((ge.rows + ntb - 1) / ntb) * nfb;
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
  } else if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < stages; ++i) {
        mbar_init(&s.full[i], 1);
        mbar_init(&s.empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&s.tfull[i], 1);
        mbar_init(&s.tempty[i], 4);  // one lane of each epilogue warp
      }
      mbar_init(&s.drain, 1);
      s.abort = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(&s.tmem_base, W_TMEM_COLS);
    tmem_relinquish();
  } else if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&tmT);
    tma_prefetch_desc(&tmT2);
    tma_prefetch_desc(&tmW0);
    tma_prefetch_desc(&tmW1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = s.tmem_base;
  const int nk = (p.K + WB_K - 1) / WB_K;
  const int tiles = s.tile_start[p.num_groups];
  const int ks = choose_ksplit(tiles, gridDim.x, nk, p.max_ksplit);
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.ksplit_out != nullptr) *p.ksplit_out = ks;
  const int total = tiles * ks;
  volatile int* abort_flag = &s.abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint64_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok && !p.test_stall; u += gridDim.x) {
        const WtUnit wu = wt_unit(s, p, u, ks, nk, ntb);
        const int tok_row = (p.a_rows_from_out ? wu.grp.out_row0 : wu.grp.a_row0) + wu.tb * ntb;
        const CUtensorMap* mT = (wu.grp.expert == p.shared_slab) ? &tmT2 : &tmT;
        const int wrow = wu.grp.expert * p.n_per_slab + wu.fb * FEAT;
        for (int kb = wu.kb0; kb < wu.kb1; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&s.full[stage], stage_bytes);
          armed |= 1ull << stage;
          armed_phase = (armed_phase & ~(1ull << stage)) | (static_cast<uint64_t>(phase) << stage);
          uint8_t* sw = ring + stage * stage_bytes;
          uint8_t* st = sw + W_W_BYTES;
          const int kc = kb * WB_K;
          if (EPI == EPI_SWIGLU) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              tma_load_2d(sw + (2 * i) * 2048, &tmW0, kc, wrow + 16 * i, &s.full[stage]);
              tma_load_2d(sw + (2 * i + 1) * 2048, &tmW1, kc, wrow + 16 * i, &s.full[stage]);
            }
          } else {
            tma_load_2d(sw, &tmW0, kc, wrow, &s.full[stage]);
          }
          tma_load_2d(st, mT, kc, tok_row, &s.full[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
        int never = 0;
        for (int i = 0; i < stages; ++i)
          if (armed & (1ull << i)) mbar_wait(&s.full[i], static_cast<uint32_t>((armed_phase >> i) & 1ull), &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++local) {
        const WtUnit wu = wt_unit(s, p, u, ks, nk, ntb);
        const int ntr = (wu.nt + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(128, ntr);
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * W_ACC_COLS;
        for (int kb = wu.kb0; kb < wu.kb1; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w_base = smem_u32(ring + stage * stage_bytes);
          const uint32_t t_base = w_base + W_W_BYTES;
#pragma unroll
          for (int kk = 0; kk < WB_K / 16; ++kk)
            tc_mma_f16(d_tmem, smem_desc_sw128(w_base + kk * 32), smem_desc_sw128(t_base + kk * 32), idesc,
                       (kb > wu.kb0 || kk > 0) ? 1u : 0u);
          tc_commit(&s.empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&s.tfull[acc]);
      }
      tc_commit(&s.drain);
      int never = 0;
      mbar_wait(&s.drain, 0, &never);
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3;  // TMEM lane quarter of this warp
    __nv_bfloat16* tbuf = tbufs + (warp - 2) * (W_TBUF / 2);
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      const WtUnit wu = wt_unit(s, p, u, ks, nk, ntb);
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
      const uint32_t tbase = tmem + acc * W_ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);
      const int nchunks = (wu.nt + WT_CHUNK - 1) / WT_CHUNK;
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[WT_CHUNK];
        tmem_ld_32x32b_x16(tbase + c * WT_CHUNK, r);
        tmem_ld_wait();
        wt_store_chunk<EPI>(p, wu.grp, wu.split, wu.fb * FEAT, wu.tb * ntb, q, lane, c, r, ks, tbuf);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, W_TMEM_COLS);
  }
}

template <int EPI>
cudaError_t launch_wt_epi(const CUtensorMap& mT, const CUtensorMap& mT2, const CUtensorMap& mW0,
                          const CUtensorMap& mW1, const TcParams& p, int grid, int ntb, int stages, size_t smem,
                          int64_t max_group_rows, cudaStream_t stream) {
  static uint64_t attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(grouped_gemm_wt_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemLimit));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  grouped_gemm_wt_kernel<EPI><<<grid, W_THREADS, smem, stream>>>(mT, mT2, mW0, mW1, p, ntb, stages);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.max_ksplit <= 1) return e;
  dim3 fgrid((p.N + 1023) / 1024, static_cast<unsigned>(max_group_rows), p.num_groups);
  splitk_finalize_kernel<EPI><<<fgrid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Weights-as-M launch: `p` is filled by the dispatcher.  The token block (TMA
// box height and largest MMA N) is the largest group's row count rounded up
// to 16, at most 256; the ring takes as many stages as fit.
cudaError_t launch_grouped_gemm_wt(const GemmArgs& a, const gemm::TcParams& p, int num_sms, cudaStream_t stream) {
  int64_t g = a.max_group_rows < 256 ? a.max_group_rows : 256;
  if (g < 1) g = 1;
  const int ntb = static_cast<int>((g + 15) & ~int64_t(15));
  const size_t stage_bytes = W_W_BYTES + static_cast<size_t>(ntb) * WB_K * 2;
  int stages = static_cast<int>((kSmemLimit - kWtFixed) / stage_bytes);
  if (stages > W_MAX_STAGES) stages = W_MAX_STAGES;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = stages * stage_bytes + kWtFixed;
  CUtensorMap mT, mT2, mW0, mW1;
  if (!make_map(&mT, a.a, a.a_rows, a.K, ntb)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    if (!make_map(&mT2, a.a_shared, a.a_shared_rows, a.K, ntb)) return cudaErrorInvalidValue;
  } else {
    mT2 = mT;
  }
  const int wbox = a.epilogue == EPI_SWIGLU ? 16 : 128;
  if (!make_map(&mW0, a.b0, a.b_rows, a.K, wbox)) return cudaErrorInvalidValue;
  if (a.epilogue == EPI_SWIGLU) {
    if (!make_map(&mW1, a.b1, a.b_rows, a.K, wbox)) return cudaErrorInvalidValue;
  } else {
    mW1 = mW0;
  }
  const int grid = num_sms > 0 ? num_sms : 1;
  switch (a.epilogue) {
    case EPI_SWIGLU:
      return launch_wt_epi<EPI_SWIGLU>(mT, mT2, mW0, mW1, p, grid, ntb, stages, smem, a.max_group_rows, stream);
    case EPI_GELU_BIAS:
      return launch_wt_epi<EPI_GELU_BIAS>(mT, mT2, mW0, mW1, p, grid, ntb, stages, smem, a.max_group_rows, stream);
    case EPI_BIAS:
      return launch_wt_epi<EPI_BIAS>(mT, mT2, mW0, mW1, p, grid, ntb, stages, smem, a.max_group_rows, stream);
    case EPI_NONE:
      return launch_wt_epi<EPI_NONE>(mT, mT2, mW0, mW1, p, grid, ntb, stages, smem, a.max_group_rows, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace moe
