// quant_math.cuh -- the per-group arithmetic of the 1 x 128 / 128 x 128 E4M3
// quantizers ("Lesson 13: DeepSeek DeepGEMM core architecture and Hopper FP8
// kernel breakdown", Fig. 13-1 and the answer to Q1), shared by the quantizer
// kernels and the GEMM's quantizing epilogue so that both give the same bits.
//
// Per group:  amax = max |x|;  s = fl32(amax / 448) (optionally rounded up to
// a power of two);  code = E4M3_RNE_satfinite(fl32(x / s)).  The quotient is
// the correctly rounded FP32 value, computed from the correctly rounded
// reciprocal and two FMA corrections (Markstein's theorem; see quantize.cu).
#pragma once

#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dg.h"

namespace dg {

constexpr float kE4M3Max = 448.0f;
constexpr float kFastDivMin = 7.8886090522101181e-31f;  // 2^-100

// Smallest power of two >= a (a >= 0, finite), from the FP32 bits.
__device__ __forceinline__ float pow2_round_up(float a) {
  const uint32_t b = __float_as_uint(a);
  const uint32_t e = (b >> 23) & 0xFFu, m = b & 0x7FFFFFu;
  if (m == 0) return a;  // zero or already a power of two
  if (e != 0) return __uint_as_float((e + 1u) << 23);
  // subnormal: next power of two of the mantissa field (may reach 2^-126)
  return __uint_as_float(1u << (32 - __clz(m - 1u)));
}

__device__ __forceinline__ float group_scale(float amax, int flags) {
  float s = __fdiv_rn(amax, kE4M3Max);
  if (flags & DG_SCALE_POW2) s = pow2_round_up(s);
  return s;
}

// RN(x / s) from y = RN(1/s); valid for s >= 2^-100 (see the file comment).
__device__ __forceinline__ float div_by_scale(float x, float s, float y) {
  const float q0 = x * y;
  const float q1 = fmaf(fmaf(-s, q0, x), y, q0);
  return fmaf(fmaf(-s, q1, x), y, q1);
}

// Four E4M3 codes of the quotients q[0..3], little-endian in 32 bits.  The
// sign of each code is taken from the dividend v (the scale is positive), so
// values that round to zero, -0.0 included, keep their sign.
__device__ __forceinline__ uint32_t pack_codes(const float q[4], const float v[4]) {
  const uint32_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE, __NV_E4M3);
  // top byte of each dividend (sign + 7 exponent bits), masked to the sign
  const uint32_t t01 = __byte_perm(__float_as_uint(v[0]), __float_as_uint(v[1]), 0x73);
  const uint32_t t23 = __byte_perm(__float_as_uint(v[2]), __float_as_uint(v[3]), 0x73);
  const uint32_t signs = __byte_perm(t01, t23, 0x5410) & 0x80808080u;
  return (lo | (hi << 16)) | signs;
}

// Codes of v[0..3] divided by the group scale.
__device__ __forceinline__ uint32_t encode4(const float v[4], float s, float y, bool fast) {
  if (s == 0.0f) return 0u;  // all-zero group
  float q[4];
  if (fast) {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = div_by_scale(v[i], s, y);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __fdiv_rn(v[i], s);
  }
  return pack_codes(q, v);
}

}  // namespace dg
