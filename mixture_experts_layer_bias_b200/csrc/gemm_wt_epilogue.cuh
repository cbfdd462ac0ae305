// Epilogue shared by the weights-as-M GEMM kernels (one-CTA and CTA-pair):
// TMEM lanes hold weight rows (output features), TMEM columns hold tokens.
#pragma once

#include "gemm_common.cuh"

namespace moe {
namespace gemm {

constexpr int WT_CHUNK = 16;  // tokens per epilogue chunk (one 32x32b.x16 TMEM load)

// Epilogue of one 16-token chunk of a weights-as-M tile (a CTA holds 128
// weight rows in its TMEM lanes and the tile's tokens in its columns):
// r[j] is the accumulator of this thread's lane for token tok0 + chunk*16 + j
// of group `grp`.  feat0 is the first output feature of this CTA's 128 rows
// (SwiGLU: 64 features, gate and up interleaved in blocks of 16 rows).
// Stores go through `tbuf` (1 KB per warp, 16-byte aligned) so that global
// stores are 16-byte pieces of output rows; split-K partials go straight out.
template <int EPI>
__device__ __forceinline__ void wt_store_chunk(const TcParams& p, const GroupEntry& grp, int split, int feat0,
                                               int tok0, int q, int lane, int chunk, const uint32_t (&r)[WT_CHUNK],
                                               int ks, __nv_bfloat16* tbuf) {
  const int N = p.N;
  const int t0 = tok0 + chunk * WT_CHUNK;  // first token of the chunk inside the group
  const int64_t row0 = static_cast<int64_t>(grp.out_row0) + t0;
  const int64_t sbase = static_cast<int64_t>(grp.expert) * N;
  const int tlim = min(WT_CHUNK, grp.rows - t0);  // valid tokens in this chunk
  if (EPI == EPI_SWIGLU) {
    const int blk = q * 2 + (lane >> 4);  // 16-row block of this CTA's weight rows
    const bool is_up = blk & 1;
    const int fbase = feat0 + (blk >> 1) * 16;
    const int f = fbase + (lane & 15);
    const bool fvalid = f < N;
    if (ks > 1) {
      if (!fvalid) return;
      float* base = p.partial + (static_cast<int64_t>(split) * p.out_rows + row0) * p.pcols + (is_up ? N : 0) + f;
#pragma unroll
      for (int j = 0; j < WT_CHUNK; ++j)
        if (j < tlim) base[static_cast<int64_t>(j) * p.pcols] = __uint_as_float(r[j]);
      return;
    }
    float sg = 1.0f, su = 1.0f;
    if (p.scale0 != nullptr && fvalid) {
      sg = __ldg(p.scale0 + sbase + f);
      su = __ldg(p.scale1 + sbase + f);
    }
    // lanes 0-15: h for 16 features x 16 tokens -> tbuf[token][feature] (16 x 16 bf16)
#pragma unroll
    for (int j = 0; j < WT_CHUNK; ++j) {
      const float mine = __uint_as_float(r[j]);
      const float up = __shfl_xor_sync(0xFFFFFFFFu, mine, 16);
      if (!is_up) {
        const float g = mine * sg;
        tbuf[j * 16 + lane] = __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * (up * su));
      }
    }
    __syncwarp();
    // 16 tokens x 32 bytes = 32 pieces of 16 bytes, one per lane
    const int tok = lane >> 1, sub = lane & 1;
    const int fo = fbase + sub * 8;
    if (tok < tlim && fo + 8 <= N)
      stg16(static_cast<__nv_bfloat16*>(p.out) + (row0 + tok) * N + fo,
            *reinterpret_cast<const uint4*>(tbuf + tok * 16 + sub * 8));
    __syncwarp();
  } else {
    const int fbase = feat0 + q * 32;
    const int f = fbase + lane;
    if (ks > 1) {
      if (f >= N) return;
      float* base = p.partial + (static_cast<int64_t>(split) * p.out_rows + row0) * p.pcols + f;
#pragma unroll
      for (int j = 0; j < WT_CHUNK; ++j)
        if (j < tlim) base[static_cast<int64_t>(j) * p.pcols] = __uint_as_float(r[j]);
      return;
    }
    const bool fvalid = f < N;
    const float sc = (p.scale0 != nullptr && fvalid) ? __ldg(p.scale0 + sbase + f) : 1.0f;
    const float bi = ((EPI == EPI_GELU_BIAS || EPI == EPI_BIAS) && fvalid) ? __ldg(p.bias + sbase + f) : 0.0f;
    if (p.out_f32) {
      // fp32 output (router logits): 32 lanes write 128 contiguous bytes per token
      if (!fvalid) return;
#pragma unroll
      for (int j = 0; j < WT_CHUNK; ++j)
        if (j < tlim) static_cast<float*>(p.out)[(row0 + j) * N + f] = __uint_as_float(r[j]) * sc + bi;
      return;
    }
#pragma unroll
    for (int j = 0; j < WT_CHUNK; ++j) {
      float z = __uint_as_float(r[j]) * sc + bi;
      if (EPI == EPI_GELU_BIAS) z = 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
      tbuf[j * 32 + lane] = __float2bfloat16_rn(z);
    }
    __syncwarp();
    // 16 tokens x 64 bytes = 64 pieces of 16 bytes, two per lane
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int piece = lane + 32 * h;
      const int tok = piece >> 2, sub = piece & 3;
      const int fo = fbase + sub * 8;
      if (tok < tlim && fo + 8 <= N)
        stg16(static_cast<__nv_bfloat16*>(p.out) + (row0 + tok) * N + fo,
              *reinterpret_cast<const uint4*>(tbuf + tok * 32 + sub * 8));
    }
    __syncwarp();
  }
}

}  // namespace gemm
}  // namespace moe
