// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dg.h"

namespace dg {

// ---------------------------------------------------------------- quantizers
int launch_quantize_1x128(const void *x, int x_dtype, int64_t batch, int64_t M,
                          int64_t K, int64_t ld_x, uint8_t *q, int64_t ld_q,
                          float *sf, int64_t ld_sf, int flags,
                          cudaStream_t stream, int num_sms);

int launch_quantize_128x1(const void *x, int x_dtype, int64_t K, int64_t M, int64_t ld_x,
                          uint8_t *q, int64_t ld_q, float *sf, int64_t ld_sf, int flags,
                          cudaStream_t stream);

int launch_quantize_128x128(const float *w, int64_t G, int64_t N, int64_t K,
                            uint8_t *q, float *sf, int flags,
                            cudaStream_t stream);

// Launch attribute for programmatic dependent launch (the kernel waits for
// the previous grid on the device, after its own set-up).
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a = {};
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// ---------------------------------------------------------------- GEMM
// kDenseCluster: dense tiles every one split `splits` ways along K, the splits
// of a tile forming one thread-block cluster that reduces through
// distributed shared memory (decode-sized shapes; no workspace).
// kDenseAcc: dense tiles with D = C + A B^T (an FP32 C added before the BF16
// rounding); the host picks it for a dense launch that has a C.
// kKGrouped: the groups split K; group g computes its own FP32
// D[g] = C[g] + A_g B_g^T over its K segment, with 1x128 scales on both
// operands (one B scale per column and K block).
// kDenseUE8M0 / kMaskedUE8M0: the dense and masked tiles with power-of-two
// scales given as packed UE8M0 codes, applied by the tensor cores
// (block-scaled MMA): the tile accumulates in TMEM over all of K and the
// promotion warps only drain it for the epilogue.
// kDenseQuant: dense tiles whose epilogue quantizes D: each row's 128-column
// groups go out as E4M3 codes with one FP32 scale, as the 1x128 quantizer
// would write them from the BF16 result.
// kDensePair: dense 256-row tiles computed by the two CTAs of a cluster with
// cta_group::2 MMAs (each CTA loads its 128 rows of A and half of the B tile,
// so each SM moves two thirds of the single-CTA form's operand bytes).
enum Sched : int {
  kDense = 0, kContiguous = 1, kMasked = 2, kDenseCluster = 3, kDenseAcc = 4, kKGrouped = 5,
  kDenseUE8M0 = 6, kMaskedUE8M0 = 7, kDenseQuant = 8, kDensePair = 9
};

// Operand layouts of D = A * B^T ("DeepGEMM architecture deep dive",
// section 3: sm_100 supports NT, TN, NN and TT).  The letters say how A and B
// are used: N as stored, T transposed.  NT: A [M][K], B [N][K] (both
// K-major); NN: B stored [K][N]; TN: A [K][M] and B [K][N]; TT: A [K][M].
// An operand stored with K outermost is MN-major in shared memory.
enum Layout : int { kLayoutNT = 0, kLayoutNN = 1, kLayoutTN = 2, kLayoutTT = 3 };
__host__ __device__ constexpr bool a_mn_major(int layout) {
  return layout == kLayoutTN || layout == kLayoutTT;
}
__host__ __device__ constexpr bool b_mn_major(int layout) {
  return layout == kLayoutNN || layout == kLayoutTN;
}

// The tile schedule (work list, row validity, epilogue) a schedule follows.
__host__ __device__ constexpr int base_sched(int sched) {
  return (sched == kDenseUE8M0 || sched == kDenseQuant || sched == kDensePair) ? kDense
         : sched == kMaskedUE8M0                        ? kMasked
                                                        : sched;
}
__host__ __device__ constexpr bool is_ue8m0(int sched) {
  return sched == kDenseUE8M0 || sched == kMaskedUE8M0;
}

// Kernel parameters besides the two tensor maps.  Row coordinates are inside
// one "slab": the whole of A for dense and contiguous, one expert's M_max rows
// for masked.  The k-grouped schedule's own fields share storage with fields
// it does not use (so the struct, and every other schedule's code, stays as
// it was).
struct GemmParams {
  const float *sfa;      // MN-major alpha: [slab][K/128][ld_sfa]; UE8M0: packed
                         // int32 words [slab][ceil(K/512)][ld_sfa]
  int64_t ld_sfa;
  const float *sfb;      // beta: [group][ceil(N/128)][K/128]; k-grouped:
                         // MN-major [K/128][ld_sfb], one scale per column;
                         // UE8M0: int32 words [group][ceil(K/512)][ld_sfb]
                         // per row of B
  union {
    uint16_t *d;         // BF16 output [slab][rows][N]
    float *d_f32;        // k-grouped: FP32 output [group][rows][N]
    uint8_t *dq;         // quantizing epilogue: E4M3 codes [rows][N]
  };
  union {
    const float *c;      // dense D = C + A B^T: FP32 C [rows][N]; k-grouped:
                         // [group][rows][N] (nullptr: none)
    float *sfd;          // quantizing epilogue: MN-major scales [N/128][ld_sfd]
  };
  const int32_t *m_indices;  // contiguous: expert per row (-1 = padding)
  union {
    const int32_t *masked_m;  // masked: valid rows per expert
    const int32_t *k_sizes;   // k-grouped: K of each group, multiples of 128
  };
  int *status;           // device status word (first error wins)
  float *ws;             // split-K partials (nullptr: no split)
  union {
    uint32_t *ws_ticket;  // split-K arrival counters, one per output tile
    int64_t ld_sfb;       // k-grouped and UE8M0: row stride of the B scales
    int64_t ld_sfd;       // quantizing epilogue: row stride of D's scales
  };
  int rows;              // dense: M; contiguous: M_total; masked: M_max
  int n, k;
  int groups;            // experts (1 for dense)
  int num_m_blocks;      // ceil(rows / 128)
  int num_n_blocks;      // ceil(n / BN)
  int num_k_blocks;      // k / 128
  int splits;            // K splits of the split tiles (1 = none)
  int full_tiles;        // dense: tiles (in raster order) computed whole before
                         // the remaining ones, each split `splits` ways
  int a_box_rows;        // rows of A per TMA load: 128, or 64 when M <= 64
  int q_flags;           // quantizing epilogue: DG_SCALE_FP32 or DG_SCALE_POW2
  int starve_it;         // test hook: the K-block iteration whose loads CTA 0's
                         // producer leaves out (-1: none; set by launch_fp8_gemm)
};

struct GemmConfig {
  int block_n;
  int stages;
  int splits;
  int num_sms;
  int smem_bytes;
};

// Host entry of the GEMM: picks a config, encodes tensor maps, launches.
// `layout` (kLayoutNT .. kLayoutTT) selects how A and B are stored; layouts
// other than NT serve the dense and k-grouped schedules.
int launch_fp8_gemm(int sched, const uint8_t *A, const uint8_t *B,
                    GemmParams p, cudaStream_t stream, int num_sms,
                    size_t ws_bytes, void *ws, int layout = kLayoutNT);

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int num_sms);

// ---------------------------------------------------------------- device state
struct DeviceInfo {
  int ok;            // 1 when the device is usable (sm_100)
  int num_sms;
  int max_smem_optin;
  int *status;       // device address of the status word
};

// Per-device properties (cached); returns nullptr on a CUDA error.
const DeviceInfo *device_info();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t,
                                  void *, const cuuint64_t *, const cuuint64_t *,
                                  const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

int effective_num_sms();

}  // namespace dg
