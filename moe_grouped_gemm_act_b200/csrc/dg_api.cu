// dg_api.cu -- the C ABI (include/dg.h): argument validation, per-device state
// and dispatch to the kernels.  No entry point allocates device memory or
// synchronizes, except dg_get_device_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "dg.h"
#include "internal.h"
#include "ptx.cuh"

namespace dg {

__device__ int g_status = 0;

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_info_once[kMaxDevices];
int g_sm_cap = 0;  // dg_set_num_sms; 0 = all

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

const DeviceInfo *device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_info_once[dev], [dev] {
    DeviceInfo &d = g_info[dev];
    int major = 0, sms = 0, smem = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.ok = (major == 10) ? 1 : 0;
    d.num_sms = sms;
    d.max_smem_optin = smem;
    // resolve the status word's device address (this also loads the module,
    // so later calls can be captured into a CUDA graph)
    void *st = nullptr;
    if (cudaGetSymbolAddress(&st, g_status) != cudaSuccess) d.ok = 0;
    d.status = static_cast<int *>(st);
  });
  return &g_info[dev];
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

int effective_num_sms() {
  const DeviceInfo *d = device_info();
  if (!d) return 0;
  const int cap = g_sm_cap;
  return (cap > 0 && cap < d->num_sms) ? cap : d->num_sms;
}

namespace {

// Common checks for every launch: a usable sm_100 device.
int check_device() {
  const DeviceInfo *d = device_info();
  if (!d) return DG_ERR_CUDA;
  if (!d->ok) return DG_ERR_UNSUPPORTED_ARCH;
  return DG_OK;
}

int check_gemm_common(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                      const uint8_t *B, const float *sfb, const void *D,
                      int64_t rows, int64_t N, int64_t K) {
  if (rows < 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
  if (rows == 0) return DG_OK;  // nothing is read or written
  if (!A || !sfa || !B || !sfb || !D) return DG_ERR_INVALID_ARG;
  if (ld_sfa < rows || ld_sfa <= 0) return DG_ERR_INVALID_ARG;
  if (rows > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  if (ld_sfa % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(D) || !aligned16(sfb))
    return DG_ERR_ALIGNMENT;
  return DG_OK;
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" {

const char *dg_status_string(int status) {
  switch (status) {
    case DG_OK: return "ok";
    case DG_ERR_INVALID_ARG: return "invalid argument";
    case DG_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case DG_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
    case DG_ERR_CUDA: return "CUDA error";
    case DG_ERR_WORKSPACE: return "workspace missing or too small";
    case DG_ERR_TIMEOUT: return "a pipeline wait on the device timed out";
    case DG_ERR_DEVICE_DATA: return "invalid index, count, size or scale data on the device";
    default: return "unknown status";
  }
}

int dg_get_mk_alignment_for_contiguous_layout(void) { return 128; }

int64_t dg_get_tma_aligned_size(int64_t n, int elem_bytes) {
  if (n < 0 || !(elem_bytes == 1 || elem_bytes == 2 || elem_bytes == 4 || elem_bytes == 8))
    return -1;
  const int64_t per = 16 / elem_bytes;
  return (n + per - 1) / per * per;
}

int dg_set_num_sms(int n) {
  g_sm_cap = n > 0 ? n : 0;
  return DG_OK;
}

int dg_get_num_sms(void) { return effective_num_sms(); }

int dg_quantize_1x128(const void *x, int x_dtype, int64_t batch, int64_t M, int64_t K,
                      int64_t ld_x, uint8_t *q, int64_t ld_q, float *sf, int64_t ld_sf,
                      int flags, dg_stream_t stream) {
  if (!x || !q || !sf) return DG_ERR_INVALID_ARG;
  if (x_dtype != DG_DTYPE_F32 && x_dtype != DG_DTYPE_BF16) return DG_ERR_INVALID_ARG;
  if (flags & ~DG_SCALE_POW2) return DG_ERR_INVALID_ARG;
  if (batch < 1 || M < 0 || K <= 0 || K % 128 != 0) return DG_ERR_INVALID_ARG;
  if (ld_x < K || ld_q < K || ld_sf < M) return DG_ERR_INVALID_ARG;
  const int esz = x_dtype == DG_DTYPE_F32 ? 4 : 2;
  if ((ld_x * esz) % 16 != 0 || ld_q % 16 != 0 || ld_sf % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return DG_ERR_ALIGNMENT;
  int rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  return launch_quantize_1x128(x, x_dtype, batch, M, K, ld_x, q, ld_q, sf, ld_sf, flags,
                               reinterpret_cast<cudaStream_t>(stream), effective_num_sms());
}

int dg_quantize_128x1(const void *x, int x_dtype, int64_t K, int64_t M, int64_t ld_x,
                      uint8_t *q, int64_t ld_q, float *sf, int64_t ld_sf, int flags,
                      dg_stream_t stream) {
  if (!x || !q || !sf) return DG_ERR_INVALID_ARG;
  if (x_dtype != DG_DTYPE_F32 && x_dtype != DG_DTYPE_BF16) return DG_ERR_INVALID_ARG;
  if (flags & ~DG_SCALE_POW2) return DG_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 128 != 0) return DG_ERR_INVALID_ARG;
  if (ld_x < M || ld_q < M || ld_sf < M) return DG_ERR_INVALID_ARG;
  if (ld_sf % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return DG_ERR_ALIGNMENT;
  int rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  return launch_quantize_128x1(x, x_dtype, K, M, ld_x, q, ld_q, sf, ld_sf, flags,
                               reinterpret_cast<cudaStream_t>(stream));
}

int dg_quantize_128x128(const float *w, int64_t G, int64_t N, int64_t K, uint8_t *q,
                        float *sf, int flags, dg_stream_t stream) {
  if (!w || !q || !sf) return DG_ERR_INVALID_ARG;
  if (flags & ~DG_SCALE_POW2) return DG_ERR_INVALID_ARG;
  if (G < 1 || N < 0 || K <= 0 || K % 128 != 0) return DG_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned16(sf)) return DG_ERR_ALIGNMENT;
  int rc = check_device();
  if (rc) return rc;
  if (N == 0) return DG_OK;
  return launch_quantize_128x128(w, G, N, K, q, sf, flags,
                                 reinterpret_cast<cudaStream_t>(stream));
}

size_t dg_fp8_gemm_nt_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  int sms = effective_num_sms();
  if (sms <= 0) sms = 148;  // no usable device: size for a full B200
  return gemm_workspace_size(M, N, K, sms);
}

int dg_fp8_gemm_nt(const uint8_t *A, const float *sfa, int64_t ld_sfa, const uint8_t *B,
                   const float *sfb, void *D, int64_t M, int64_t N, int64_t K,
                   void *workspace, size_t workspace_bytes, dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M, N, K);
  if (rc) return rc;
  if (workspace && !aligned16(workspace)) return DG_ERR_ALIGNMENT;
  if (!workspace) workspace_bytes = 0;
  rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.d = static_cast<uint16_t *>(D);
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = 1;
  return launch_fp8_gemm(kDense, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), workspace_bytes, workspace);
}

namespace {

// D = A * B^T with A and B stored as `layout` says (the transposed forms keep
// K outermost for the operand they transpose; its row stride, M or N bytes,
// must be a multiple of 16 for the tensor memory accelerator).
int fp8_gemm_layout(int layout, const uint8_t *A, const float *sfa, int64_t ld_sfa,
                    const uint8_t *B, const float *sfb, void *D, int64_t M, int64_t N, int64_t K,
                    void *workspace, size_t workspace_bytes, dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M, N, K);
  if (rc) return rc;
  if (a_mn_major(layout) && M % 16 != 0) return DG_ERR_ALIGNMENT;
  if (b_mn_major(layout) && N % 16 != 0) return DG_ERR_ALIGNMENT;
  if (workspace && !aligned16(workspace)) return DG_ERR_ALIGNMENT;
  if (!workspace) workspace_bytes = 0;
  rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.d = static_cast<uint16_t *>(D);
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = 1;
  return launch_fp8_gemm(kDense, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), workspace_bytes, workspace, layout);
}

}  // namespace

int dg_fp8_gemm_nn(const uint8_t *A, const float *sfa, int64_t ld_sfa, const uint8_t *B,
                   const float *sfb, void *D, int64_t M, int64_t N, int64_t K,
                   void *workspace, size_t workspace_bytes, dg_stream_t stream) {
  return fp8_gemm_layout(kLayoutNN, A, sfa, ld_sfa, B, sfb, D, M, N, K, workspace,
                         workspace_bytes, stream);
}

int dg_fp8_gemm_tn(const uint8_t *A, const float *sfa, int64_t ld_sfa, const uint8_t *B,
                   const float *sfb, void *D, int64_t M, int64_t N, int64_t K,
                   void *workspace, size_t workspace_bytes, dg_stream_t stream) {
  return fp8_gemm_layout(kLayoutTN, A, sfa, ld_sfa, B, sfb, D, M, N, K, workspace,
                         workspace_bytes, stream);
}

int dg_fp8_gemm_tt(const uint8_t *A, const float *sfa, int64_t ld_sfa, const uint8_t *B,
                   const float *sfb, void *D, int64_t M, int64_t N, int64_t K,
                   void *workspace, size_t workspace_bytes, dg_stream_t stream) {
  return fp8_gemm_layout(kLayoutTT, A, sfa, ld_sfa, B, sfb, D, M, N, K, workspace,
                         workspace_bytes, stream);
}

int dg_fp8_gemm_nt_quantize(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                            const uint8_t *B, const float *sfb, uint8_t *Dq, float *sfd,
                            int64_t ld_sfd, int64_t M, int64_t N, int64_t K, int flags,
                            dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, Dq, M, N, K);
  if (rc) return rc;
  if (flags & ~DG_SCALE_POW2) return DG_ERR_INVALID_ARG;
  if (N % 128 != 0) return DG_ERR_INVALID_ARG;
  if (M > 0 && (!sfd || ld_sfd < M)) return DG_ERR_INVALID_ARG;
  if (ld_sfd % 4 != 0) return DG_ERR_ALIGNMENT;
  if (sfd && !aligned16(sfd)) return DG_ERR_ALIGNMENT;
  rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.dq = Dq;
  p.sfd = sfd;
  p.ld_sfd = ld_sfd;
  p.q_flags = flags;
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = 1;
  return launch_fp8_gemm(kDenseQuant, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr);
}

int dg_fp8_gemm_nt_accumulate(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                              const uint8_t *B, const float *sfb, const float *C, void *D,
                              int64_t M, int64_t N, int64_t K, void *workspace,
                              size_t workspace_bytes, dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M, N, K);
  if (rc) return rc;
  if (M > 0 && !C) return DG_ERR_INVALID_ARG;
  if (C && !aligned16(C)) return DG_ERR_ALIGNMENT;
  if (workspace && !aligned16(workspace)) return DG_ERR_ALIGNMENT;
  if (!workspace) workspace_bytes = 0;
  rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.d = static_cast<uint16_t *>(D);
  p.c = C;
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = 1;
  return launch_fp8_gemm(kDense, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), workspace_bytes, workspace);
}

int dg_m_grouped_fp8_gemm_nt_contiguous(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                                        const uint8_t *B, const float *sfb, void *D,
                                        const int32_t *m_indices, int64_t M_total,
                                        int64_t N, int64_t K, int G, dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M_total, N, K);
  if (rc) return rc;
  if (!m_indices || G < 1) return DG_ERR_INVALID_ARG;
  if (M_total % 128 != 0) return DG_ERR_INVALID_ARG;
  if (!aligned16(m_indices)) return DG_ERR_ALIGNMENT;
  rc = check_device();
  if (rc) return rc;
  if (M_total == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.d = static_cast<uint16_t *>(D);
  p.m_indices = m_indices;
  p.rows = static_cast<int>(M_total);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = G;
  return launch_fp8_gemm(kContiguous, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr);
}

int dg_m_grouped_fp8_gemm_nt_masked(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                                    const uint8_t *B, const float *sfb, void *D,
                                    const int32_t *masked_m, int G, int64_t M_max,
                                    int64_t N, int64_t K, dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M_max, N, K);
  if (rc) return rc;
  if (!masked_m || G < 1 || G > 1024 || M_max < 1) return DG_ERR_INVALID_ARG;
  rc = check_device();
  if (rc) return rc;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.d = static_cast<uint16_t *>(D);
  p.masked_m = masked_m;
  p.rows = static_cast<int>(M_max);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = G;
  return launch_fp8_gemm(kMasked, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr);
}

namespace {

int k_grouped(int layout, const uint8_t *A, const float *sfa, int64_t ld_sfa, const uint8_t *B,
              const float *sfb, int64_t ld_sfb, const float *C, float *D,
              const int32_t *k_sizes, int G, int64_t M, int64_t N, int64_t K,
              dg_stream_t stream) {
  int rc = check_gemm_common(A, sfa, ld_sfa, B, sfb, D, M, N, K);
  if (rc) return rc;
  if (a_mn_major(layout) && M % 16 != 0) return DG_ERR_ALIGNMENT;
  if (b_mn_major(layout) && N % 16 != 0) return DG_ERR_ALIGNMENT;
  if (G < 1 || G > 1024) return DG_ERR_INVALID_ARG;
  if (M == 0) return DG_OK;
  if (!k_sizes || ld_sfb < N) return DG_ERR_INVALID_ARG;
  if (ld_sfb % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(k_sizes) || (C && !aligned16(C))) return DG_ERR_ALIGNMENT;
  rc = check_device();
  if (rc) return rc;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = sfa;
  p.ld_sfa = ld_sfa;
  p.sfb = sfb;
  p.ld_sfb = ld_sfb;
  p.d_f32 = D;
  p.c = C;
  p.k_sizes = k_sizes;
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = G;
  return launch_fp8_gemm(kKGrouped, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr, layout);
}

}  // namespace

int dg_k_grouped_fp8_gemm_nt_contiguous(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                                        const uint8_t *B, const float *sfb, int64_t ld_sfb,
                                        const float *C, float *D, const int32_t *k_sizes,
                                        int G, int64_t M, int64_t N, int64_t K,
                                        dg_stream_t stream) {
  return k_grouped(kLayoutNT, A, sfa, ld_sfa, B, sfb, ld_sfb, C, D, k_sizes, G, M, N, K,
                   stream);
}

int dg_k_grouped_fp8_gemm_tn_contiguous(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                                        const uint8_t *B, const float *sfb, int64_t ld_sfb,
                                        const float *C, float *D, const int32_t *k_sizes,
                                        int G, int64_t M, int64_t N, int64_t K,
                                        dg_stream_t stream) {
  return k_grouped(kLayoutTN, A, sfa, ld_sfa, B, sfb, ld_sfb, C, D, k_sizes, G, M, N, K,
                   stream);
}

namespace {

// Checks shared by the UE8M0 GEMMs (packed int32 scale words, four K groups
// each, for the rows of A and of B).
int check_gemm_ue8m0(const uint8_t *A, const int32_t *sfa, int64_t ld_sfa, const uint8_t *B,
                     const int32_t *sfb, int64_t ld_sfb, const void *D, int64_t rows,
                     int64_t N, int64_t K) {
  if (rows < 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
  if (rows == 0) return DG_OK;
  if (!A || !sfa || !B || !sfb || !D) return DG_ERR_INVALID_ARG;
  if (ld_sfa < rows || ld_sfb < N) return DG_ERR_INVALID_ARG;
  if (rows > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  if (ld_sfa % 4 != 0 || ld_sfb % 4 != 0) return DG_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb) || !aligned16(D))
    return DG_ERR_ALIGNMENT;
  return DG_OK;
}

}  // namespace

int dg_fp8_gemm_nt_ue8m0(const uint8_t *A, const int32_t *sfa, int64_t ld_sfa,
                         const uint8_t *B, const int32_t *sfb, int64_t ld_sfb, void *D,
                         int64_t M, int64_t N, int64_t K, dg_stream_t stream) {
  int rc = check_gemm_ue8m0(A, sfa, ld_sfa, B, sfb, ld_sfb, D, M, N, K);
  if (rc) return rc;
  rc = check_device();
  if (rc) return rc;
  if (M == 0) return DG_OK;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = reinterpret_cast<const float *>(sfa);
  p.ld_sfa = ld_sfa;
  p.sfb = reinterpret_cast<const float *>(sfb);
  p.ld_sfb = ld_sfb;
  p.d = static_cast<uint16_t *>(D);
  p.rows = static_cast<int>(M);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = 1;
  return launch_fp8_gemm(kDenseUE8M0, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr);
}

int dg_m_grouped_fp8_gemm_nt_masked_ue8m0(const uint8_t *A, const int32_t *sfa,
                                          int64_t ld_sfa, const uint8_t *B,
                                          const int32_t *sfb, int64_t ld_sfb, void *D,
                                          const int32_t *masked_m, int G, int64_t M_max,
                                          int64_t N, int64_t K, dg_stream_t stream) {
  int rc = check_gemm_ue8m0(A, sfa, ld_sfa, B, sfb, ld_sfb, D, M_max, N, K);
  if (rc) return rc;
  if (!masked_m || G < 1 || G > 1024 || M_max < 1) return DG_ERR_INVALID_ARG;
  rc = check_device();
  if (rc) return rc;
  GemmParams p{};
  p.status = device_info()->status;
  p.sfa = reinterpret_cast<const float *>(sfa);
  p.ld_sfa = ld_sfa;
  p.sfb = reinterpret_cast<const float *>(sfb);
  p.ld_sfb = ld_sfb;
  p.d = static_cast<uint16_t *>(D);
  p.masked_m = masked_m;
  p.rows = static_cast<int>(M_max);
  p.n = static_cast<int>(N);
  p.k = static_cast<int>(K);
  p.groups = G;
  return launch_fp8_gemm(kMaskedUE8M0, A, B, p, reinterpret_cast<cudaStream_t>(stream),
                         effective_num_sms(), 0, nullptr);
}

int dg_get_device_status(dg_stream_t stream, int *status) {
  if (!status) return DG_ERR_INVALID_ARG;
  if (!device_info()) return DG_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int h = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&h, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DG_ERR_CUDA;
  *status = h;
  return DG_OK;
}

}  // extern "C"
