// ue8m0.cu -- the packed UE8M0 scale layout and its C entry point.
//
// UE8M0 ("Lesson 13: DeepSeek DeepGEMM core architecture and Hopper FP8
// kernel breakdown", Fig. 13-1 text: newer versions accept it in place of
// FP32 scales) is an unsigned 8-bit exponent e standing for 2^(e - 127).  On
// sm_100 the LHS scales go to the GEMM as four UE8M0 values packed into one
// 32-bit integer, in the transposed, TMA-aligned layout ("DeepGEMM
// architecture deep dive", section 3).
//
// For a power-of-two FP32 scale the UE8M0 code is the FP32 exponent field,
// so packing is a pure bit operation: word (p, i) gathers the exponent bytes
// of K groups 4p .. 4p + 3 of row i, group 4p + t in bits 8t .. 8t + 7.  The
// transform is a small HBM stream (4 bytes read and 1 written per scale): one
// thread per output word, consecutive threads on consecutive rows i, so every
// load and store of a warp is one contiguous 128-byte segment.
#include <cuda_runtime.h>

#include <cstdint>

#include "dg.h"
#include "internal.h"
#include "ptx.cuh"

namespace dg {

namespace {

constexpr int kPackThreads = 256;
constexpr int kMaxGridY = 65535;

// The scale is +0 or a positive normal power of two exactly when its FP32 bit
// pattern is the exponent field alone and that field is not the all-ones
// (inf/NaN) value.
__device__ __forceinline__ uint32_t ue8m0_code(float s, bool &bad) {
  const uint32_t bits = __float_as_uint(s);
  const uint32_t e = (bits >> 23) & 0xFFu;
  bad |= bits != (e << 23) || e == 0xFFu;
  return e;
}

// sf: FP32 [batch][kg][ld_sf]; packed: int32 [batch][words][ld_packed].
// grid.x covers the rows, grid.y strides over (batch, word) pairs.
__global__ void __launch_bounds__(kPackThreads)
pack_ue8m0_kernel(const float *__restrict__ sf, int64_t rows, int64_t kg, int64_t ld_sf,
                  int64_t pairs, int64_t words, uint32_t *__restrict__ packed,
                  int64_t ld_packed, int *status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x;
  if (i >= rows) return;
  bool bad = false;
  for (int64_t bw = blockIdx.y; bw < pairs; bw += gridDim.y) {
    const int64_t b = bw / words;
    const int64_t p = bw - b * words;
    const float *src = sf + (b * kg + 4 * p) * ld_sf + i;
    const int64_t left = kg - 4 * p;  // >= 1
    uint32_t word = ue8m0_code(__ldg(src), bad);
    if (left > 1) word |= ue8m0_code(__ldg(src + ld_sf), bad) << 8;
    if (left > 2) word |= ue8m0_code(__ldg(src + 2 * ld_sf), bad) << 16;
    if (left > 3) word |= ue8m0_code(__ldg(src + 3 * ld_sf), bad) << 24;
    packed[bw * ld_packed + i] = word;
  }
  if (bad) record_status(status, DG_ERR_DEVICE_DATA);
}

// 128 x 128 block scales of B, one word per row of B: sf FP32
// [groups][nb][kg] (the quantizer's row-major block scales), packed int32
// [groups][words][ld_packed]; word (g, p, n) holds block (n / 128)'s groups
// 4p .. 4p + 3.  One thread per output word, consecutive threads on
// consecutive rows (the 128 rows of a block read the same four scales).
__global__ void __launch_bounds__(kPackThreads)
pack_ue8m0_blocks_kernel(const float *__restrict__ sf, int64_t n, int64_t nb, int64_t kg,
                         int64_t pairs, int64_t words, uint32_t *__restrict__ packed,
                         int64_t ld_packed, int *status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x;
  if (i >= n) return;
  bool bad = false;
  for (int64_t gw = blockIdx.y; gw < pairs; gw += gridDim.y) {
    const int64_t g = gw / words;
    const int64_t p = gw - g * words;
    const float *src = sf + (g * nb + i / 128) * kg + 4 * p;
    const int64_t left = kg - 4 * p;  // >= 1
    uint32_t word = ue8m0_code(__ldg(src), bad);
    if (left > 1) word |= ue8m0_code(__ldg(src + 1), bad) << 8;
    if (left > 2) word |= ue8m0_code(__ldg(src + 2), bad) << 16;
    if (left > 3) word |= ue8m0_code(__ldg(src + 3), bad) << 24;
    packed[gw * ld_packed + i] = word;
  }
  if (bad) record_status(status, DG_ERR_DEVICE_DATA);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace dg

extern "C" int dg_pack_ue8m0(const float *sf, int64_t batch, int64_t M, int64_t Kg,
                             int64_t ld_sf, int32_t *packed, int64_t ld_packed,
                             dg_stream_t stream) {
  using namespace dg;
  if (batch < 1 || M < 0 || Kg < 1) return DG_ERR_INVALID_ARG;
  if (ld_sf < M || ld_packed < M) return DG_ERR_INVALID_ARG;
  if (M == 0) return DG_OK;
  if (!sf || !packed) return DG_ERR_INVALID_ARG;
  if (ld_sf % 4 != 0 || ld_packed % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(sf) || !aligned16(packed)) return DG_ERR_ALIGNMENT;
  const DeviceInfo *d = device_info();
  if (!d) return DG_ERR_CUDA;
  if (!d->ok) return DG_ERR_UNSUPPORTED_ARCH;
  const int64_t words = (Kg + 3) / 4;
  const int64_t pairs = batch * words;
  const int64_t blocks_x = (M + kPackThreads - 1) / kPackThreads;
  if (blocks_x > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  const dim3 grid(static_cast<unsigned>(blocks_x),
                  static_cast<unsigned>(pairs < kMaxGridY ? pairs : kMaxGridY));
  pack_ue8m0_kernel<<<grid, kPackThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      sf, M, Kg, ld_sf, pairs, words, reinterpret_cast<uint32_t *>(packed), ld_packed,
      d->status);
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

extern "C" int dg_pack_ue8m0_128x128(const float *sf, int64_t G, int64_t N, int64_t Kg,
                                     int32_t *packed, int64_t ld_packed, dg_stream_t stream) {
  using namespace dg;
  if (G < 1 || N < 0 || Kg < 1 || ld_packed < N) return DG_ERR_INVALID_ARG;
  if (N == 0) return DG_OK;
  if (!sf || !packed) return DG_ERR_INVALID_ARG;
  if (ld_packed % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(sf) || !aligned16(packed)) return DG_ERR_ALIGNMENT;
  const DeviceInfo *d = device_info();
  if (!d) return DG_ERR_CUDA;
  if (!d->ok) return DG_ERR_UNSUPPORTED_ARCH;
  const int64_t words = (Kg + 3) / 4;
  const int64_t pairs = G * words;
  const int64_t blocks_x = (N + kPackThreads - 1) / kPackThreads;
  if (blocks_x > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  const dim3 grid(static_cast<unsigned>(blocks_x),
                  static_cast<unsigned>(pairs < kMaxGridY ? pairs : kMaxGridY));
  pack_ue8m0_blocks_kernel<<<grid, kPackThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      sf, N, (N + 127) / 128, Kg, pairs, words, reinterpret_cast<uint32_t *>(packed), ld_packed,
      d->status);
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}
