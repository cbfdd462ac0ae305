// Per-row E4M3 codes of bf16 activation rows (device helpers shared by the
// row-coding kernels and the one-CTA permutation that folds the coded row
// gather of tiny batches).  The two codings (W8A8 one-term codes with scale
// amax / 448; two-term codes x * 2^k = c1 + c2 with a power-of-two row scale)
// are described in quant.cu.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace coding {

constexpr int kCodeWarps = 8;  // warps of a CTA that codes a row (T = 256)

// Two finite float32 values -> their E4M3 codes (round to nearest even,
// saturating at +-448), first value in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_finite(float a, float b) {
  return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3) & 0xFFFFu;
}

// The same for any values, a NaN giving 0x7F.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint32_t q = e4m3x2_finite(a, b);
  if (isnan(a)) q = (q & 0xFF00u) | 0x7Fu;
  if (isnan(b)) q = (q & 0x00FFu) | 0x7F00u;
  return q;
}

// Magnitude of the finite E4M3 code in the low byte of c, exactly: its
// exponent and mantissa bits placed at the bottom of a float's exponent field
// and the top of its mantissa give the value times 2^-120 (an E4M3 subnormal
// becomes a float subnormal, with the same mantissa), and one multiply by
// 2^120 restores it.
__device__ __forceinline__ float e4m3_magnitude(uint32_t c) {
  return __uint_as_float((c & 0x7Fu) << 20) * 0x1p120f;
}

// Largest |x| of bf16 values kept as bit patterns: the magnitude bits of a
// bf16 (sign cleared) order like the values, with +inf = 0x7F80 above every
// finite value and NaNs above it, so two 16-bit unsigned maxima per 32-bit
// word track the row's maximum and whether it holds an infinity or a NaN.
__device__ __forceinline__ uint32_t absmax_bits2(uint32_t acc, uint32_t w) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w & 0x7FFF7FFFu));
  return r;
}

__device__ __forceinline__ uint32_t absmax_bits8(uint32_t acc, const uint4& w) {
  return absmax_bits2(absmax_bits2(absmax_bits2(absmax_bits2(acc, w.x), w.y), w.z), w.w);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// A row's 16-byte pieces held by one of T threads (a warp, or the whole CTA):
// pieces tid, tid + T, ... up to kVec of them stay in registers, so the row
// is read from memory once; pieces beyond T * kVec (rows longer than the
// launch's choice of T allows) are read again when coded.
constexpr int kVec = 8;

template <int T>
struct RowPieces {
  uint4 v[kVec];
};

// Loads the thread's pieces and reduces max |x| and the NaN / non-finite
// flags over the T threads.
template <int T>
__device__ __forceinline__ void row_load_amax(const __nv_bfloat16* __restrict__ src, int d, int tid,
                                              RowPieces<T>& rp, float& amax, bool& nan, bool& nonfinite) {
  uint32_t acc = 0;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int c = (tid + i * T) * 8;
    rp.v[i] = c < d ? ldg16(src + c) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kVec; ++i) acc = absmax_bits8(acc, rp.v[i]);  // zero pieces past the row change nothing
  for (int c = (tid + kVec * T) * 8; c < d; c += T * 8) acc = absmax_bits8(acc, ldg16(src + c));
  uint32_t bits = __reduce_max_sync(0xFFFFFFFFu, max(acc & 0xFFFFu, acc >> 16));
  if (T > 32) {
    __shared__ uint32_t wm[kCodeWarps];
    if ((tid & 31) == 0) wm[tid >> 5] = bits;
    __syncthreads();
    bits = wm[0];
#pragma unroll
    for (int i = 1; i < T / 32; ++i) bits = max(bits, wm[i]);
    __syncthreads();  // the next row's maxima reuse wm
  }
  amax = __uint_as_float(bits << 16);
  nan = bits > 0x7F80u;
  nonfinite = bits >= 0x7F80u;
}

// W8A8 scale: amax / 448 (1 for an all-zero row or a row holding a NaN).
__device__ __forceinline__ float w8a8_scale(float amax, bool nan) {
  return (!nan && amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// Two-term multiplier 2^k (0 for a row with a non-finite value, whose codes
// are all zero) and scale 2^-k (NaN for such a row).
__device__ __forceinline__ float two_term_mult(float amax, bool nonfinite, float& scale) {
  if (nonfinite) {
    scale = __int_as_float(0x7FC00000);
    return 0.0f;
  }
  int k = 0;
  if (amax > 0.0f) {
    int ex;
    const float f = frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
    k = (f <= 0.875f ? 9 : 8) - ex;     // 448 = 0.875 * 2^9
    k = max(-126, min(126, k));
  }
  scale = __int_as_float((127 - k) << 23);
  return __int_as_float((127 + k) << 23);
}

// W8A8 codes of 8 bf16 values for the row scale s, in memory order.
__device__ __forceinline__ uint2 encode8_w8a8(const uint4& w, float s) {
  float f[8];
  bf16x8_to_f32(w, f);
  uint32_t q[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) q[j] = e4m3x2(__fdiv_rn(f[2 * j], s), __fdiv_rn(f[2 * j + 1], s));
  return make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
}

// Two-term codes of 8 bf16 values for the multiplier m, each term in memory
// order (zero codes for m = 0: a row with a non-finite value).
__device__ __forceinline__ void encode8_two_term(const uint4& w, float m, uint2& t1, uint2& t2) {
  if (m == 0.0f) {
    t1 = t2 = make_uint2(0, 0);
    return;
  }
  float f[8];
  bf16x8_to_f32(w, f);
  uint32_t a[4], b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float v0 = f[2 * j] * m, v1 = f[2 * j + 1] * m;  // finite, |v| <= 448
    a[j] = e4m3x2_finite(v0, v1);
    // c1 carries v's sign (or is zero), so v - c1 = v - copysign(|c1|, v)
    b[j] = e4m3x2_finite(v0 - copysignf(e4m3_magnitude(a[j]), v0), v1 - copysignf(e4m3_magnitude(a[j] >> 8), v1));
  }
  t1 = make_uint2(a[0] | (a[1] << 16), a[2] | (a[3] << 16));
  t2 = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

// Scale (and two-term multiplier) of a row from its maximum.
__device__ __forceinline__ void row_scale(int terms, float amax, bool nan, bool nonfinite, float& s, float& m) {
  if (terms == 2) {
    m = two_term_mult(amax, nonfinite, s);
  } else {
    s = w8a8_scale(amax, nan);
    m = 1.0f;
  }
}

// Codes of the row piece starting at column c: term codes to dst[c..] (and
// dst[d + c..] for two terms).
__device__ __forceinline__ void code_piece(const uint4& w, uint8_t* __restrict__ dst, int d, int c, int terms,
                                           float s, float m) {
  if (terms == 2) {
    uint2 t1, t2;
    encode8_two_term(w, m, t1, t2);
    *reinterpret_cast<uint2*>(dst + c) = t1;
    *reinterpret_cast<uint2*>(dst + d + c) = t2;
  } else {
    *reinterpret_cast<uint2*>(dst + c) = encode8_w8a8(w, s);
  }
}

// Codes of one row of d bf16 values (d % 8 == 0) by T threads (thread `tid`):
// terms = 1 (d codes) or 2 (2d codes: first terms, then second terms); the
// row's scale goes to *scale.
template <int T>
__device__ __forceinline__ void code_row(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                                         float* __restrict__ scale, int d, int terms, int tid) {
  RowPieces<T> rp;
  float amax, s, m;
  bool nan, nonfinite;
  row_load_amax<T>(src, d, tid, rp, amax, nan, nonfinite);
  row_scale(terms, amax, nan, nonfinite, s, m);
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int c = (tid + i * T) * 8;
    if (c < d) code_piece(rp.v[i], dst, d, c, terms, s, m);
  }
  for (int c = (tid + kVec * T) * 8; c < d; c += T * 8) code_piece(ldg16(src + c), dst, d, c, terms, s, m);
  if (tid == 0) *scale = s;
}


}  // namespace coding
}  // namespace moe
