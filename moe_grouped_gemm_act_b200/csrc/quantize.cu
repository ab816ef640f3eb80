// quantize.cu -- FP8 E4M3 quantizers: 1 x 128 activation groups and 128 x 128
// weight blocks ("Lesson 13: DeepSeek DeepGEMM core architecture and Hopper
// FP8 kernel breakdown", Fig. 13-1 and the answer to Q1).
//
// Both are bandwidth-bound streaming kernels.  The 1 x 128 kernel gives one
// warp one 128-element group at a time: each lane loads 16 bytes (4 FP32 or
// 4 BF16 through an 8-byte load), the warp reduces |x| with shuffles, the
// scale is the correctly rounded FP32 quotient amax / 448 (optionally rounded
// up to a power of two), every element is divided by it with correctly
// rounded FP32 division and converted to E4M3 with round-to-nearest-even and
// saturation.  Each warp keeps kItems groups in flight for memory-level
// parallelism.  Scales go to the MN-major layout the GEMM reads.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dg.h"
#include "internal.h"

namespace dg {

namespace {

constexpr float kE4M3Max = 448.0f;

// Smallest power of two >= a (a >= 0, finite), from the FP32 bits.
__device__ __forceinline__ float pow2_round_up(float a) {
  uint32_t b = __float_as_uint(a);
  const uint32_t e = (b >> 23) & 0xFFu, m = b & 0x7FFFFFu;
  if (m == 0) return a;  // zero or already a power of two
  if (e != 0) return __uint_as_float((e + 1u) << 23);
  // subnormal: next power of two of the mantissa field (may reach 2^-126)
  const uint32_t p = 1u << (32 - __clz(m - 1u));
  return __uint_as_float(p);
}

__device__ __forceinline__ float group_scale(float amax, int flags) {
  float s = __fdiv_rn(amax, kE4M3Max);
  if (flags & DG_SCALE_POW2) s = pow2_round_up(s);
  return s;
}

// Four E4M3 codes of v[0..3] / s, packed little-endian into 32 bits.
__device__ __forceinline__ uint32_t encode4(const float v[4], float s) {
  if (s == 0.0f) return 0u;  // all-zero group
  float q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = __fdiv_rn(v[i], s);
  const uint32_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE, __NV_E4M3);
  uint32_t r = lo | (hi << 16);
  // keep the sign of values that round to zero
  uint32_t sg = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) sg |= ((__float_as_uint(q[i]) >> 31) << (8 * i + 7));
  return r | sg;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <typename T>
__device__ __forceinline__ void load4(const T *p, float v[4]);

template <>
__device__ __forceinline__ void load4<float>(const float *p, float v[4]) {
  const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p,
                                                     float v[4]) {
  const uint2 t = __ldcs(reinterpret_cast<const uint2 *>(p));
  v[0] = __uint_as_float(t.x << 16);
  v[1] = __uint_as_float(t.x & 0xFFFF0000u);
  v[2] = __uint_as_float(t.y << 16);
  v[3] = __uint_as_float(t.y & 0xFFFF0000u);
}

constexpr int kItems = 4;  // groups in flight per warp

template <typename T>
__global__ void __launch_bounds__(256)
quantize_1x128_kernel(const T *__restrict__ x, int64_t batch, int64_t M,
                      int64_t Kg, int64_t ld_x, uint8_t *__restrict__ q,
                      int64_t ld_q, float *__restrict__ sf, int64_t ld_sf,
                      int flags) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t total = batch * M * Kg;  // items = (b, i, g), g fastest

  for (int64_t base = warp * kItems; base < total; base += nwarps * kItems) {
    float v[kItems][4];
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      const int64_t it = base + u;
      if (it < total) {
        const int64_t row = it / Kg, g = it - row * Kg;  // row = b * M + i
        load4(x + row * ld_x + g * 128 + lane * 4, v[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      const int64_t it = base + u;
      if (it >= total) break;
      const int64_t row = it / Kg, g = it - row * Kg;
      float a = fmaxf(fmaxf(fabsf(v[u][0]), fabsf(v[u][1])),
                      fmaxf(fabsf(v[u][2]), fabsf(v[u][3])));
      a = warp_max(a);
      const float s = group_scale(a, flags);
      const uint32_t codes = encode4(v[u], s);
      *reinterpret_cast<uint32_t *>(q + row * ld_q + g * 128 + lane * 4) = codes;
      if (lane == 0) {
        const int64_t b = row / M, i = row - b * M;
        sf[(b * Kg + g) * ld_sf + i] = s;
      }
    }
  }
}

// One CTA of 256 threads per 128 x 128 block.  Thread t covers columns
// 4 (t % 32) .. +3 of rows t / 32 + 8 j, j < 16.
__global__ void __launch_bounds__(256)
quantize_128x128_kernel(const float *__restrict__ w, int64_t N, int64_t K,
                        uint8_t *__restrict__ q, float *__restrict__ sf,
                        int flags) {
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
  a = red[lane & 7];
  a = warp_max(a);
  const float s = group_scale(a, flags);
  if (t == 0) sf[(b * Nb + nb) * Kg + g] = s;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int64_t r = nb * 128 + wid + 8 * j;
    if (r < N) *reinterpret_cast<uint32_t *>(dst + r * K + col) = encode4(v[j], s);
  }
}

}  // namespace

int launch_quantize_1x128(const void *x, int x_dtype, int64_t batch, int64_t M,
                          int64_t K, int64_t ld_x, uint8_t *q, int64_t ld_q,
                          float *sf, int64_t ld_sf, int flags,
                          cudaStream_t stream, int num_sms) {
  const int64_t Kg = K / 128;
  const int64_t items = batch * M * Kg;
  const int threads = 256;
  const int64_t warps_needed = (items + kItems - 1) / kItems;
  int64_t blocks = (warps_needed * 32 + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;  // 8 x 256 threads / SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (x_dtype == DG_DTYPE_F32) {
    quantize_1x128_kernel<float><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        static_cast<const float *>(x), batch, M, Kg, ld_x, q, ld_q, sf, ld_sf, flags);
  } else {
    quantize_1x128_kernel<__nv_bfloat16>
        <<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), batch, M, Kg, ld_x, q, ld_q, sf,
            ld_sf, flags);
  }
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

int launch_quantize_128x128(const float *w, int64_t G, int64_t N, int64_t K,
                            uint8_t *q, float *sf, int flags,
                            cudaStream_t stream) {
  const int64_t blocks = G * ((N + 127) / 128) * (K / 128);
  if (blocks > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  quantize_128x128_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      w, N, K, q, sf, flags);
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

}  // namespace dg
