// Grouped expert GEMM on CTA pairs (tcgen05 .cta_group::2), weights as the
// M operand.
//
// Same operation as the one-CTA kernel (jsqmd.com "第11章 MoE模型推理" 11.1.2:
// the S*K expert forwards run grouped by expert; plumephp.com "MoE 混合专家推理",
// "sequence expert": one large GEMM per expert), arranged for ragged groups:
//
//   D[feature, token] = sum_k W[expert][feature, k] * A[token, k]
//
// A pair of CTAs (one cluster) owns a tile of 256 weight rows (M, 128 in each
// CTA's shared memory and TMEM lanes) by up to 256 tokens (N, any multiple of
// 16: the last token block of a group is padded by at most 15 rows, instead of
// up to 127 or 255 when tokens are the M operand).  The two CTAs each load
// half of the tokens; one thread of the even CTA issues the MMAs for both.
// Per CTA and K-step of 64 the ring holds 16 KB of weights and 16 KB of
// tokens, so six stages fit and each CTA moves 2/3 of the bytes the one-CTA
// 128 x 256 tile moves for the same work.
//
// SwiGLU: a CTA's 128 weight rows are 64 gate and 64 up rows interleaved in
// blocks of 16 (gate f..f+15, up f..f+15, ...), so in every 32-lane TMEM
// quarter lanes 0-15 hold gate and lanes 16-31 the up accumulator of the same
// 16 features, and one shuffle pairs them in the epilogue.
//
// Roles per CTA (192 threads): warp 0 TMA producer (both CTAs; completion
// counted on the even CTA's barrier), warp 1 TMEM owner and, in the even CTA,
// MMA issuer, warps 2-5 epilogue (both CTAs: tcgen05.ld, activation, stores
// or split-K partial sums).  Waits are bounded in time as in the one-CTA
// kernel.  No load uses cluster multicast; only the MMA completion signal
// (tcgen05.commit) reaches both CTAs.
#include "gemm_wt_epilogue.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int P_BK = 64;
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = 128 * P_BK * 2;  // 128 weight rows per CTA
constexpr int P_B_BYTES = 128 * P_BK * 2;  // up to 128 token rows per CTA
constexpr int P_STAGE = P_A_BYTES + P_B_BYTES;
constexpr int P_TOK = 256;       // tokens per pair tile (MMA N <= 256)
constexpr int P_ACC_COLS = 256;  // one accumulator buffer
constexpr int P_TMEM_COLS = 512;
constexpr int P_THREADS = 192;
constexpr uint32_t kLeaderTx = 2 * P_STAGE;  // bytes both CTAs deliver per stage

struct PairCtl {
  uint64_t full[P_STAGES];
  uint64_t empty[P_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[kMaxGroups + 1];
};

// per epilogue warp: one 16-token x 32-feature bf16 tile, transposed through
// shared memory so that global stores are 16-byte pieces of output rows
constexpr int P_TBUF = 16 * 32 * 2;
constexpr size_t kPairCtlBytes = (sizeof(PairCtl) + 127) & ~size_t(127);  // keeps the buffers 128-byte aligned
constexpr size_t kPairSmem = P_STAGES * P_STAGE + kPairCtlBytes + 4 * P_TBUF + 1024;

template <int EPI>
struct PairShape {
  static constexpr int FEAT = EPI == EPI_SWIGLU ? 128 : 256;  // output features per pair tile
};

struct PairUnit {
  GroupEntry grp;
  int fb, tb, split, kb0, kb1, nt;  // nt = tokens of this block (<= 256)
};

__device__ __forceinline__ PairUnit pair_unit(const PairCtl& s, const TcParams& p, int u, int ks, int nk) {
  PairUnit pu;
  const int tt = u / ks;
  pu.split = u - tt * ks;
  int lo = 0, hi = p.num_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= tt)
      lo = mid;
    else
      hi = mid;
  }
  pu.grp = group_at(p, lo);
  const int ntb = (pu.grp.rows + P_TOK - 1) / P_TOK;
  const int local = tt - s.tile_start[lo];
  pu.fb = local / ntb;
  pu.tb = local - pu.fb * ntb;
  pu.nt = min(P_TOK, pu.grp.rows - pu.tb * P_TOK);
  pu.kb0 = static_cast<int>((static_cast<int64_t>(pu.split) * nk) / ks);
  pu.kb1 = static_cast<int>((static_cast<int64_t>(pu.split + 1) * nk) / ks);
  return pu;
}

__device__ __forceinline__ bool wait_timed_pair(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never);
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmT2,
                             const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                             TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PairCtl& s = *reinterpret_cast<PairCtl*>(ring + P_STAGES * P_STAGE);
  __nv_bfloat16* tbufs = reinterpret_cast<__nv_bfloat16*>(ring + P_STAGES * P_STAGE + kPairCtlBytes);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  constexpr int FEAT = PairShape<EPI>::FEAT;
  const int nfb = (p.N + FEAT - 1) / FEAT;

  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.num_groups; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < p.num_groups) {
        const GroupEntry ge = group_at(p, g);
        if (group_ok(ge, p))
          tiles = ((ge.rows + P_TOK - 1) / P_TOK) * nfb;
        else if (ge.rows != 0 && rank == 0)
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
      for (int i = 0; i < P_STAGES; ++i) {
        mbar_init(&s.full[i], 1);
        mbar_init(&s.empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&s.tfull[i], 1);
        mbar_init(&s.tempty[i], 8);  // one lane of each epilogue warp of both CTAs
      }
      mbar_init(&s.drain, 1);
      s.abort = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc_pair(&s.tmem_base, P_TMEM_COLS);
    tmem_relinquish_pair();
  } else if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&tmT);
    tma_prefetch_desc(&tmT2);
    tma_prefetch_desc(&tmW0);
    tma_prefetch_desc(&tmW1);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote signal
  tc_fence_after();

  const uint32_t tmem = s.tmem_base;
  const int nk = (p.K + P_BK - 1) / P_BK;
  const int tiles = s.tile_start[p.num_groups];
  const int ks = choose_ksplit(tiles, nclusters, nk, p.max_ksplit);
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.ksplit_out != nullptr) *p.ksplit_out = ks;
  const int total = tiles * ks;
  volatile int* abort_flag = &s.abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int u = cluster; u < total && ok; u += nclusters) {
        const PairUnit pu = pair_unit(s, p, u, ks, nk);
        const int ntr = (pu.nt + 15) & ~15;
        const int half = ntr >> 1;
        const int tok_row = (p.a_rows_from_out ? pu.grp.out_row0 : pu.grp.a_row0) + pu.tb * P_TOK +
                            static_cast<int>(rank) * half;
        const CUtensorMap* mT = (pu.grp.expert == p.shared_slab) ? &tmT2 : &tmT;
        const int wrow = pu.grp.expert * p.n_per_slab + pu.fb * FEAT + static_cast<int>(rank) * (FEAT / 2);
        for (int kb = pu.kb0; kb < pu.kb1; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) {
            mbar_arrive_expect_tx(&s.full[stage], kLeaderTx);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t bar = mapa_shared(smem_u32(&s.full[stage]), 0);
          uint8_t* sa = ring + stage * P_STAGE;
          uint8_t* sb = sa + P_A_BYTES;
          const int kc = kb * P_BK;
          if (EPI == EPI_SWIGLU) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              tma_load_2d_pair(sa + (2 * i) * 2048, &tmW0, kc, wrow + 16 * i, bar);
              tma_load_2d_pair(sa + (2 * i + 1) * 2048, &tmW1, kc, wrow + 16 * i, bar);
            }
          } else {
            tma_load_2d_pair(sa, &tmW0, kc, wrow, bar);
          }
          tma_load_2d_pair(sb, mT, kc, tok_row, bar);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
        if (rank == 0) {
          for (int i = 0; i < P_STAGES; ++i)
            if (armed & (1u << i)) wait_timed_pair(&s.full[i], (armed_phase >> i) & 1u);
        } else {
          // copies of this CTA count on the peer's barriers: give them time to land
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 2000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = cluster; u < total && ok; u += nclusters, ++local) {
        const PairUnit pu = pair_unit(s, p, u, ks, nk);
        const int ntr = (pu.nt + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(256, ntr);
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * P_ACC_COLS;
        for (int kb = pu.kb0; kb < pu.kb1; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + stage * P_STAGE);
          const uint32_t b_base = a_base + P_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < P_BK / 16; ++kk)
            tc_mma_f16_pair(d_tmem, smem_desc_sw128(a_base + kk * 32), smem_desc_sw128(b_base + kk * 32), idesc,
                            (kb > pu.kb0 || kk > 0) ? 1u : 0u);
          tc_commit_pair_mask(&s.empty[stage], 0x3);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mask(&s.tfull[acc], 0x3);
      }
      tc_commit_pair(&s.drain);
      wait_timed_pair(&s.drain, 0);
      if (!ok) {
        *abort_flag = 1;
        report(p.status, MOE_STATUS_TIMEOUT, MOE_CNT_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3;  // TMEM lane quarter of this warp
    int local = 0;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&s.tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&s.tempty[1]), 0);
    for (int u = cluster; u < total; u += nclusters, ++local) {
      const PairUnit pu = pair_unit(s, p, u, ks, nk);
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
      const uint32_t tbase = tmem + acc * P_ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);
      const int nchunks = (pu.nt + WT_CHUNK - 1) / WT_CHUNK;
      const int feat0 = pu.fb * FEAT + static_cast<int>(rank) * (FEAT / 2);
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[WT_CHUNK];
        tmem_ld_32x32b_x16(tbase + c * WT_CHUNK, r);
        tmem_ld_wait();
        wt_store_chunk<EPI>(p, pu.grp, pu.split, feat0, pu.tb * P_TOK, q, lane, c, r, ks,
                            tbufs + (warp - 2) * (P_TBUF / 2));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the even CTA's MMAs read this CTA's shared memory and TMEM until here
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, P_TMEM_COLS);
  }
}

template <int EPI>
cudaError_t launch_pair_epi(const CUtensorMap& mT, const CUtensorMap& mT2, const CUtensorMap& mW0,
                            const CUtensorMap& mW1, const TcParams& p, int grid, int64_t max_group_rows,
                            cudaStream_t stream) {
  static uint64_t attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPairSmem));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  grouped_gemm_pair_kernel<EPI><<<grid, P_THREADS, kPairSmem, stream>>>(mT, mT2, mW0, mW1, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.max_ksplit <= 1) return e;
  dim3 fgrid((p.N + 1023) / 1024, static_cast<unsigned>(max_group_rows), p.num_groups);
  splitk_finalize_kernel<EPI><<<fgrid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Pair launch: `p` is filled by the dispatcher; the maps are built here
// (tokens: box 64 x 128 rows; weights: box 64 x 128 rows, or 64 x 16 rows for
// the interleaved SwiGLU gate/up blocks).
cudaError_t launch_grouped_gemm_pair(const GemmArgs& a, const gemm::TcParams& p, int num_sms, cudaStream_t stream) {
  CUtensorMap mT, mT2, mW0, mW1;
  if (!make_map(&mT, a.a, a.a_rows, a.K, 128)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    if (!make_map(&mT2, a.a_shared, a.a_shared_rows, a.K, 128)) return cudaErrorInvalidValue;
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
  int grid = num_sms & ~1;
  if (grid < 2) grid = 2;
  switch (a.epilogue) {
    case EPI_SWIGLU: return launch_pair_epi<EPI_SWIGLU>(mT, mT2, mW0, mW1, p, grid, a.max_group_rows, stream);
    case EPI_GELU_BIAS: return launch_pair_epi<EPI_GELU_BIAS>(mT, mT2, mW0, mW1, p, grid, a.max_group_rows, stream);
    case EPI_BIAS: return launch_pair_epi<EPI_BIAS>(mT, mT2, mW0, mW1, p, grid, a.max_group_rows, stream);
    case EPI_NONE: return launch_pair_epi<EPI_NONE>(mT, mT2, mW0, mW1, p, grid, a.max_group_rows, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
