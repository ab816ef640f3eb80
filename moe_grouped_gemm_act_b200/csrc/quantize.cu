// quantize.cu -- FP8 E4M3 quantizers: 1 x 128 activation groups and 128 x 128
// weight blocks ("Lesson 13: DeepSeek DeepGEMM core architecture and Hopper
// FP8 kernel breakdown", Fig. 13-1 and the answer to Q1).
//
// Per group:  amax = max |x|;  s = fl32(amax / 448) (optionally rounded up to
// a power of two);  code = E4M3_RNE_satfinite(fl32(x / s)).
//
// Both kernels are bandwidth-bound streams, so the per-element work is kept
// small.  The quotient fl32(x / s) must be the correctly rounded FP32 value
// (the codes are bit-exact); instead of a full IEEE division per element it is
// computed from the correctly rounded reciprocal y = RN(1/s), taken once per
// group, and two FMA correction steps:
//     q0 = RN(x y);  q1 = RN(q0 + RN(x - s q0) y);  q = RN(q1 + (x - s q1) y)
// The first step makes q1 a faithful approximation of x / s (relative error
// about 2^-46 before rounding); by Markstein's theorem (a faithful quotient
// plus one FMA correction with a reciprocal of relative error < 2^-24 gives
// the correctly rounded quotient, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 1990) q = RN(x / s).
// The theorem needs normal operands and no underflow: groups with
// s < 2^-100 take a plain correctly rounded division instead (for them x
// may be subnormal while x / s is not tiny); for s >= 2^-100 any subnormal x
// gives |x / s| < 2^-26, which encodes to a signed zero whatever the
// last bits.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dg.h"
#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace dg {

namespace {

template <typename T>
__device__ __forceinline__ void load4(const T *p, float v[4]);

template <>
__device__ __forceinline__ void load4<float>(const float *p, float v[4]) {
  const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float v[4]) {
  const uint2 t = __ldcs(reinterpret_cast<const uint2 *>(p));
  v[0] = __uint_as_float(t.x << 16);
  v[1] = __uint_as_float(t.x & 0xFFFF0000u);
  v[2] = __uint_as_float(t.y << 16);
  v[3] = __uint_as_float(t.y & 0xFFFF0000u);
}

// 1 x 128 groups: a warp takes 4 consecutive groups at a time, 8 lanes per
// group, 16 elements per lane.  Lane j of a group reads elements
// 32 i + 4 j .. +3 (i < 4), so each load instruction covers one contiguous
// 128-byte line per group.
template <typename T>
__global__ void __launch_bounds__(256)
quantize_1x128_kernel(const T *__restrict__ x, int64_t batch, int64_t M, int64_t Kg,
                      int64_t ld_x, uint8_t *__restrict__ q, int64_t ld_q,
                      float *__restrict__ sf, int64_t ld_sf, int flags) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 3, j = lane & 7;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t total = batch * M * Kg;  // items = (b, i, g), g fastest

  for (int64_t base = warp * 4; base < total; base += nwarps * 4) {
    const int64_t it = base + sub;
    const bool live = it < total;
    const int64_t row = live ? it / Kg : 0;  // row = b * M + i
    const int64_t g = live ? it - row * Kg : 0;
    float v[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (live) {
        load4(x + row * ld_x + g * 128 + i * 32 + j * 4, v[i]);
      } else {
        v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.0f;
      }
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      a = fmaxf(a, fmaxf(fmaxf(fabsf(v[i][0]), fabsf(v[i][1])),
                         fmaxf(fabsf(v[i][2]), fabsf(v[i][3]))));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (!live) continue;
    const float s = group_scale(a, flags);
    const bool fast = s >= kFastDivMin;
    const float y = fast ? __frcp_rn(s) : 0.0f;
    uint8_t *qrow = q + row * ld_q + g * 128 + j * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint32_t *>(qrow + i * 32) = encode4(v[i], s, y, fast);
    if (j == 0) {
      const int64_t b = row / M, r = row - b * M;
      sf[(b * Kg + g) * ld_sf + r] = s;
    }
  }
}

// Groups of 128 rows of one column: x stored [K][M] (M contiguous), the group
// of column m and K group g is x[128 g .. 128 g + 127][m] -- the 1 x 128
// groups along K of an operand stored with K outermost.  Each thread owns one
// column of one group: it loads the group's 128 values into registers (a warp
// reads 32 consecutive columns of a row: one 128-byte line for FP32), takes
// their amax, and writes the codes back row by row and the scale to
// sf[g][m] (MN-major).
template <typename T>
__global__ void __launch_bounds__(128)
quantize_128x1_kernel(const T *__restrict__ x, int64_t M, int64_t ld_x, uint8_t *__restrict__ q,
                      int64_t ld_q, float *__restrict__ sf, int64_t ld_sf, int flags) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int64_t m = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t g = blockIdx.y;
  if (m >= M) return;
  const T *src = x + g * 128 * ld_x + m;
  float v[128];
  float a = 0.0f;
#pragma unroll
  for (int r = 0; r < 128; ++r) {
    if constexpr (sizeof(T) == 4) {
      v[r] = __ldcs(reinterpret_cast<const float *>(src) + r * ld_x);
    } else {
      v[r] = __uint_as_float(static_cast<uint32_t>(
                 __ldcs(reinterpret_cast<const unsigned short *>(src) + r * ld_x)) << 16);
    }
    a = fmaxf(a, fabsf(v[r]));
  }
  const float s = group_scale(a, flags);
  const bool fast = s >= kFastDivMin;
  const float y = fast ? __frcp_rn(s) : 0.0f;
  uint8_t *dst = q + g * 128 * ld_q + m;
#pragma unroll
  for (int r = 0; r < 128; r += 4) {
    const uint32_t w = encode4(v + r, s, y, fast);
    dst[(r + 0) * ld_q] = static_cast<uint8_t>(w);
    dst[(r + 1) * ld_q] = static_cast<uint8_t>(w >> 8);
    dst[(r + 2) * ld_q] = static_cast<uint8_t>(w >> 16);
    dst[(r + 3) * ld_q] = static_cast<uint8_t>(w >> 24);
  }
  sf[g * ld_sf + m] = s;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One CTA of 256 threads per 128 x 128 block.  Thread t covers columns
// 4 (t % 32) .. +3 of rows t / 32 + 8 j, j < 16.
__global__ void __launch_bounds__(256)
quantize_128x128_kernel(const float *__restrict__ w, int64_t N, int64_t K,
                        uint8_t *__restrict__ q, float *__restrict__ sf, int flags) {
  __shared__ float red[8];
  const int64_t Kg = K / 128, Nb = (N + 127) / 128;
  const int64_t blk = blockIdx.x;
  const int64_t b = blk / (Nb * Kg);
  const int64_t nb = (blk / Kg) % Nb;
  const int64_t g = blk % Kg;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  const int64_t col = g * 128 + lane * 4;
  const float *src = w + b * N * K;
  uint8_t *dst = q + b * N * K;

  float v[16][4];
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int64_t r = nb * 128 + wid + 8 * j;
    if (r < N) {
      load4(src + r * K + col, v[j]);
    } else {
      v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0.0f;
    }
    a = fmaxf(a, fmaxf(fmaxf(fabsf(v[j][0]), fabsf(v[j][1])),
                       fmaxf(fabsf(v[j][2]), fabsf(v[j][3]))));
  }
  a = warp_max(a);
  if (lane == 0) red[wid] = a;
  __syncthreads();
  a = warp_max(red[lane & 7]);
  const float s = group_scale(a, flags);
  const bool fast = s >= kFastDivMin;
  const float y = fast ? __frcp_rn(s) : 0.0f;
  if (t == 0) sf[(b * Nb + nb) * Kg + g] = s;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int64_t r = nb * 128 + wid + 8 * j;
    if (r < N) *reinterpret_cast<uint32_t *>(dst + r * K + col) = encode4(v[j], s, y, fast);
  }
}

}  // namespace

int launch_quantize_1x128(const void *x, int x_dtype, int64_t batch, int64_t M, int64_t K,
                          int64_t ld_x, uint8_t *q, int64_t ld_q, float *sf, int64_t ld_sf,
                          int flags, cudaStream_t stream, int num_sms) {
  const int64_t Kg = K / 128;
  const int64_t items = batch * M * Kg;
  const int threads = 256;
  const int64_t warps_needed = (items + 3) / 4;
  int64_t blocks = (warps_needed * 32 + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;  // 8 x 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  // one wave of CTAs (all resident), launched as a programmatic dependent
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (x_dtype == DG_DTYPE_F32) {
    e = cudaLaunchKernelEx(&cfg, quantize_1x128_kernel<float>, static_cast<const float *>(x),
                           batch, M, Kg, ld_x, q, ld_q, sf, ld_sf, flags);
  } else {
    e = cudaLaunchKernelEx(&cfg, quantize_1x128_kernel<__nv_bfloat16>,
                           static_cast<const __nv_bfloat16 *>(x), batch, M, Kg, ld_x, q, ld_q, sf,
                           ld_sf, flags);
  }
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

int launch_quantize_128x1(const void *x, int x_dtype, int64_t K, int64_t M, int64_t ld_x,
                          uint8_t *q, int64_t ld_q, float *sf, int64_t ld_sf, int flags,
                          cudaStream_t stream) {
  const int64_t blocks_x = (M + 127) / 128;
  if (blocks_x > 0x7FFFFFFF || K / 128 > 65535) return DG_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks_x), static_cast<unsigned>(K / 128));
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (x_dtype == DG_DTYPE_F32) {
    e = cudaLaunchKernelEx(&cfg, quantize_128x1_kernel<float>, static_cast<const float *>(x), M,
                           ld_x, q, ld_q, sf, ld_sf, flags);
  } else {
    e = cudaLaunchKernelEx(&cfg, quantize_128x1_kernel<__nv_bfloat16>,
                           static_cast<const __nv_bfloat16 *>(x), M, ld_x, q, ld_q, sf, ld_sf,
                           flags);
  }
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

int launch_quantize_128x128(const float *w, int64_t G, int64_t N, int64_t K, uint8_t *q,
                            float *sf, int flags, cudaStream_t stream) {
  const int64_t blocks = G * ((N + 127) / 128) * (K / 128);
  if (blocks > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  quantize_128x128_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(w, N, K, q, sf,
                                                                             flags);
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

}  // namespace dg
