// Block quantization helpers shared by the activation quantizer and the
// GEMM's quantizing epilogue, so that both produce the same bits: packed
// bf16 magnitude maxima, the block divisor (scale, reciprocal, exact-division
// flag), x / s by one Markstein correction step (P. Markstein, IBM J. Res.
// Dev. 34(1), 1990) and the E4M3 codes.  See quant.cu for the arithmetic.
#pragma once

#include "common.cuh"

namespace fp8bw {
namespace {

constexpr uint32_t kAbsMask = 0x7FFF7FFFu;

__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// max |x| over a packed word's two halves, as a float (bf16 widened)
__device__ __forceinline__ float halves_max(uint32_t m) {
  const uint32_t lo = m & 0xFFFFu, hi = m >> 16;
  return __uint_as_float((lo > hi ? lo : hi) << 16);
}

// Larger-magnitude halves of two packed bf16 words (sign bits arbitrary:
// mask with kAbsMask before reading the magnitudes).  One instruction per
// word pair; magnitudes compare exactly as the non-negative bf16 values.
__device__ __forceinline__ uint32_t magmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t absmax8(uint4 v) {
  return umax2(umax2(v.x & kAbsMask, v.y & kAbsMask), umax2(v.z & kAbsMask, v.w & kAbsMask));
}

__device__ __forceinline__ float rcp_rn(float s) {
  float y;
  asm("rcp.rn.f32 %0, %1;" : "=f"(y) : "f"(s));
  return y;
}

// Per-block divisor: scale s, reciprocal y, and whether the block must use
// IEEE division (FP32 mode with amax < 2^-80).
struct Divisor {
  float s, y;
  bool exact;
};

template <int MODE, int FMT = FP8BW_FMT_E4M3>
__device__ __forceinline__ Divisor make_divisor(float amax) {
  Divisor d;
  d.s = block_scale<MODE, FMT>(amax);
  if (MODE == FP8BW_SCALE_POW2) {
    d.y = rcp_rn(d.s);  // exact: s is a power of two in [2^-127, 2^127]
    d.exact = false;
  } else {
    d.exact = !(amax >= 0x1p-80f);
    d.y = d.exact ? 0.0f : rcp_rn(d.s);
  }
  return d;
}

// RN(x / s) for a pair of values with per-lane divisors (s0,y0), (s1,y1):
// power-of-2 mode multiplies by the exact reciprocal, FP32 mode takes one
// Markstein step in its sign-symmetric form (the remainder is taken as
// q0*s - x and applied with -y), which gives -0 for x = -0 without a
// separate sign copy.  Blocks that need IEEE division take the slow path.
template <int MODE>
__device__ __forceinline__ float2 div2(float2 x, float2 s, float2 y) {
  if (MODE == FP8BW_SCALE_POW2) return fmul2(x, y);
  const float2 q0 = fmul2(x, y);
  const float2 r = ffma2(q0, s, make_float2(-x.x, -x.y));
  return ffma2(r, make_float2(-y.x, -y.y), q0);
}

// Scalar RN(x / s) in FP32 mode, IEEE division for a block that needs it.
__device__ __forceinline__ float div1(float x, const Divisor& d) {
  if (d.exact) return __fdiv_rn(x, d.s);
  const float q0 = __fmul_rn(x, d.y);
  const float r = __fmaf_rn(q0, d.s, -x);
  return __fmaf_rn(r, -d.y, q0);
}

template <int MODE, int FMT>
__device__ __forceinline__ uint2 quant8_fast(uint4 v, float s, float y) {
  const float2 s2 = make_float2(s, s), y2 = make_float2(y, y);
  const float2 a = div2<MODE>(make_float2(bf16lo(v.x), bf16hi(v.x)), s2, y2);
  const float2 b = div2<MODE>(make_float2(bf16lo(v.y), bf16hi(v.y)), s2, y2);
  const float2 c = div2<MODE>(make_float2(bf16lo(v.z), bf16hi(v.z)), s2, y2);
  const float2 e = div2<MODE>(make_float2(bf16lo(v.w), bf16hi(v.w)), s2, y2);
  return make_uint2(cvt_fp8x2<FMT>(a.x, a.y) | (cvt_fp8x2<FMT>(b.x, b.y) << 16),
                    cvt_fp8x2<FMT>(c.x, c.y) | (cvt_fp8x2<FMT>(e.x, e.y) << 16));
}

// Slow path (kept out of line so the fast path carries no division code).
template <int FMT>
__device__ __noinline__ uint2 quant8_exact(uint4 v, Divisor d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2];
  for (int i = 0; i < 2; ++i)
    o[i] = cvt_fp8x2<FMT>(div1(bf16lo(w[2 * i]), d), div1(bf16hi(w[2 * i]), d)) |
           (cvt_fp8x2<FMT>(div1(bf16lo(w[2 * i + 1]), d), div1(bf16hi(w[2 * i + 1]), d)) << 16);
  return make_uint2(o[0], o[1]);
}

// 8 codes of one 16-byte vector with one divisor (uniform branch per warp).
template <int MODE, int FMT = FP8BW_FMT_E4M3>
__device__ __forceinline__ uint2 quant8(uint4 v, const Divisor& d) {
  if (MODE == FP8BW_SCALE_FP32 && __any_sync(0xffffffffu, d.exact)) return quant8_exact<FMT>(v, d);
  return quant8_fast<MODE, FMT>(v, d.s, d.y);
}

struct ColCodes {
  uint32_t c0[8], c1[8];
};
struct ColWords {
  uint32_t w[32];
};

// Slow path of the column pass (a column block with amax < 2^-80).
template <int FMT>
__device__ __noinline__ ColCodes column_codes_exact(ColWords v, Divisor d0, Divisor d1) {
  ColCodes c;
  for (int i = 0; i < 8; ++i) {
    float a[4], b[4];
    for (int u = 0; u < 4; ++u) {
      a[u] = div1(bf16lo(v.w[4 * i + u]), d0);
      b[u] = div1(bf16hi(v.w[4 * i + u]), d1);
    }
    c.c0[i] = cvt_fp8x2<FMT>(a[0], a[1]) | (cvt_fp8x2<FMT>(a[2], a[3]) << 16);
    c.c1[i] = cvt_fp8x2<FMT>(b[0], b[1]) | (cvt_fp8x2<FMT>(b[2], b[3]) << 16);
  }
  return c;
}


// A 128x128 bf16 tile in shared memory as two boxes of 64 columns (128 rows
// x 128 bytes each) with the 128-byte swizzle: 16-byte chunk j of row r is
// stored at chunk j ^ (r & 7).
__device__ __forceinline__ uint32_t act_off(int box, int r, int chunk) {
  return (uint32_t)(box * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4));
}

}  // namespace
}  // namespace fp8bw
