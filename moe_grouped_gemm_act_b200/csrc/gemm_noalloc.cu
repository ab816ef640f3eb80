// gemm_noalloc.cu -- dg_fp8_gemm_nt_noalloc: the dense GEMM for callers that
// cannot allocate device memory.
//
// dg_fp8_gemm_nt takes its split-K scratch from the caller.  Some callers have
// no way to provide it: an inference runtime that reserves all of device
// memory at start-up and forbids allocation afterwards, a plugin whose host
// framework owns every buffer and only hands over inputs and outputs at
// enqueue time, or a latency-critical loop that cannot afford cudaMalloc's
// implicit device-wide synchronisation.  This entry point serves them: its
// scratch is a fixed array in this library's own device memory, allocated by
// the CUDA driver when the library's code is loaded onto a device and held
// until the process exits.
//
// Limit: the array holds kNoAllocScratchBytes (32 MiB).  A shape whose
// preferred K split needs more (dg_fp8_gemm_nt_workspace_size above that) is
// rejected with DG_ERR_WORKSPACE; shapes that do not split need no scratch.
// Every split the GEMM picks keeps split tiles x splits <= the SM count, so
// the need is at most SMs x 128 x 256 x 4 bytes plus one counter per SM: about
// 19.4 MB on a 148-SM B200, under the limit for any device of up to 256 SMs,
// where the refusal cannot happen.
//
// All calls on a device share the one array and leave their partial sums in
// it; the split-K arrival counters are cleared by every call before its
// kernel runs.  Two calls whose kernels overlap on the GPU (different streams
// without ordering between them) race on the array and may produce wrong
// results: serialise them.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "dg.h"
#include "internal.h"

namespace dg {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;

// The scratch itself.  In host code `g_noalloc_scratch` only names a
// host-side stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Per device: the resolved address, or nullptr while it is not known.  Only
// a successful lookup is kept, so a first call that failed (for instance one
// made inside a stream capture) does not disable the entry point: the next
// call tries again.
void *g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  The first call
// on a device resolves it (this also loads the array's module on that device,
// which is why that first call must not happen inside a stream capture).
int scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();  // do not leave this error for the caller's next check
      return DG_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return DG_OK;
}

}  // namespace
}  // namespace dg

extern "C" int dg_fp8_gemm_nt_noalloc(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                                      const uint8_t *B, const float *sfb, void *D, int64_t M,
                                      int64_t N, int64_t K, dg_stream_t stream) {
  using namespace dg;
  // same argument rules as dg_fp8_gemm_nt
  if (M < 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
  if (M == 0) return DG_OK;
  const size_t need = dg_fp8_gemm_nt_workspace_size(M, N, K);
  if (need > kNoAllocScratchBytes) return DG_ERR_WORKSPACE;
  void *scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != DG_OK) return rc;
  // the dense entry point validates the rest and launches with the scratch,
  // offered as exactly the bytes the size query reports, so that it picks the
  // same tile form and split as dg_fp8_gemm_nt given that workspace
  return dg_fp8_gemm_nt(A, sfa, ld_sfa, B, sfb, D, M, N, K, scratch, need > 16 ? need : 16,
                        stream);
}
