// gemm.cu -- the fine-grained block-scaled FP8 GEMM for sm_100a.
//
// Computes, per output tile of 128 rows x BN columns ("Lesson 13: DeepSeek
// DeepGEMM core architecture and Hopper FP8 kernel breakdown", Fig. 13-1):
//     acc = sum over 128-wide K blocks g of  alpha[row, g] * beta[g, col/128]
//                                            * (A_g x B_g^T)   (FP8 products)
//     D   = BF16_RNE(acc)
// with each block's FP8 partial product formed by the tensor cores and the
// scaled promotion into an FP32 accumulator done on the CUDA cores inside the
// main loop (Fig. 13-1 "promotion in the main loop"; Fig. 13-2 producer /
// consumer pipeline).  The Hopper design on that page (TMA producer warpgroup,
// WGMMA into registers, math warpgroups) is re-derived for Blackwell:
//
//   warp 0      TMA producer: one elected lane streams A [128 x 128] and
//               B [BN x 128] K blocks into a STAGES-deep shared-memory ring
//               (128-byte swizzle), completing on `full` mbarriers.
//   warp 1      MMA issuer: one lane issues 4 tcgen05.mma (kind::f8f6f4,
//               M=128, N=BN, K=32) per K block into one of two TMEM
//               accumulator buffers, then tcgen05.commit frees the smem stage
//               (`empty`) and publishes the buffer (`tmem_full`).  Each K
//               block's product starts from zero (fresh partial sum).
//   warps 4-11  promotion warpgroups: TMEM row i is read by the warp whose
//               index mod 4 is i / 32; the two warpgroups split the BN
//               columns.  Each thread owns one row and BN/2 columns: it loads
//               the partial sum with tcgen05.ld, releases the TMEM buffer
//               (`tmem_empty`) so the next block's MMA can start, and does
//               acc += partial * (alpha_row * beta) in registers.  After the
//               last K block it converts to BF16 and stores its row segment.
//
// The kernel is persistent (one CTA per SM).  All roles walk the same tile
// sequence produced by a scheduler that knows the three layouts:
//   dense       tiles of D in an M-grouped raster (L2 reuse of B);
//   contiguous  as dense over M_total, the expert of each 128-row block read
//               from the per-row index; blocks holding only padding skipped;
//   masked      per expert g, ceil(masked_m[g] / 128) row blocks x N blocks,
//               counts read on the device (launch shape independent of them).
// Dense small-M shapes may split K (units = tile x split); FP32 partials go to
// a workspace and the last-arriving CTA of a tile reduces them in split order.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "dg.h"
#include "internal.h"
#include "ptx.cuh"

namespace dg {

namespace {

constexpr int BM = 128;                 // rows per tile (one UMMA M)
constexpr int BK = 128;                 // K per block = one scale group
constexpr int kThreads = 384;           // 4 control warps + 2 promotion warpgroups
constexpr int kPromoThreads = 256;
constexpr int kPromoWarps = 8;
constexpr int kRasterGroupM = 16;       // M blocks per raster group (dense)
constexpr uint32_t kABytes = BM * BK;   // 16 KB per stage

template <int BN>
struct Layout {
  static constexpr uint32_t kBBytes = BN * BK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = (2 * BN < 32) ? 32 : 2 * BN;
};

// ------------------------------------------------------------------ scheduler
struct Tile {
  int m_blk, n_blk, split;
  int slab;     // A / D slab (expert for masked, else 0)
  int group;    // B / beta group (expert, 0 for dense)
  int k_begin, k_end;  // K blocks of this unit
};

// Returns the number of work units for this launch (dense/contiguous: tiles x
// splits; masked: from the prefix table in shared memory).
__device__ __forceinline__ int num_units(const GemmParams &p, int sched,
                                         const int *s_prefix) {
  if (sched == kMasked) return s_prefix[p.groups];
  return p.num_m_blocks * p.num_n_blocks * p.splits;
}

// Maps unit u to a tile.  Contiguous expert lookup is done separately.
__device__ __forceinline__ Tile unit_to_tile(const GemmParams &p, int sched,
                                             int u, const int *s_prefix,
                                             const int *s_mblocks) {
  Tile t;
  t.split = 0;
  t.slab = 0;
  t.group = 0;
  if (sched == kMasked) {
    // largest e with prefix[e] <= u
    int lo = 0, hi = p.groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int r = u - s_prefix[e];
    const int mb = s_mblocks[e];
    t.slab = e;
    t.group = e;
    t.n_blk = r / mb;
    t.m_blk = r - t.n_blk * mb;
  } else {
    const int s = p.splits;
    const int tile = u / s;
    t.split = u - tile * s;
    const int span = kRasterGroupM * p.num_n_blocks;
    const int grp = tile / span;
    const int first_m = grp * kRasterGroupM;
    const int gm = min(kRasterGroupM, p.num_m_blocks - first_m);
    const int r = tile - grp * span;
    t.m_blk = first_m + r % gm;
    t.n_blk = r / gm;
  }
  // K range of this split: contiguous, balanced to within one block.
  const int kb = p.num_k_blocks, s = p.splits;
  t.k_begin = (kb * t.split) / s;
  t.k_end = (kb * (t.split + 1)) / s;
  return t;
}

// Contiguous layout: the expert of a 128-row block, or -1 when the block holds
// only padding.  Whole warp; every lane returns the same value.  When
// `check` is set, a block mixing experts or holding an index >= groups records
// DG_ERR_DEVICE_DATA (rows of other experts are then not written).
__device__ __forceinline__ int block_expert(const GemmParams &p, int m_blk,
                                            bool check) {
  const int lane = threadIdx.x & 31;
  const int4 v = __ldg(reinterpret_cast<const int4 *>(p.m_indices) + m_blk * 32 + lane);
  const int vals[4] = {v.x, v.y, v.z, v.w};
  int first = 0x7FFFFFFF;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (vals[i] >= 0 && first == 0x7FFFFFFF) first = vals[i];
  // lowest lane with a valid row holds the block's first valid index
  const unsigned any = __ballot_sync(0xffffffffu, first != 0x7FFFFFFF);
  if (!any) return -1;
  const int src = __ffs(any) - 1;
  const int e = __shfl_sync(0xffffffffu, first, src);
  if (check) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) bad |= (vals[i] >= 0 && vals[i] != e);
    bad |= (e >= p.groups);
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(p.status, DG_ERR_DEVICE_DATA);
  }
  return e < p.groups ? e : -1;
}

// ------------------------------------------------------------------ the kernel
template <int BN, int STAGES, int SCHED>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
  using L = Layout<BN>;
  constexpr int W = BN / 2;  // columns per promotion thread
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(W == 8 || W == 16 || W == 32 || W == 64, "TMEM load width");

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);

  const uint32_t bar_base = base + STAGES * L::kStageBytes;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);
  uint8_t *misc = smem + STAGES * L::kStageBytes + 8 * (2 * STAGES + 5);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(misc);
  volatile int *s_abort = reinterpret_cast<volatile int *>(misc + 4);
  int *s_flag = reinterpret_cast<int *>(misc + 8);
  int *s_prefix = reinterpret_cast<int *>(misc + 16);          // [groups + 1]
  int *s_mblocks = s_prefix + (SCHED == kMasked ? p.groups + 1 : 0);  // [groups]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- setup
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kPromoWarps);
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), L::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (SCHED == kMasked) {
    if (warp == 2) {
      // prefix[e] = sum_{e' < e} ceil(clamp(masked_m[e'])/128) * n_blocks
      int running = 0;
      for (int e0 = 0; e0 < p.groups; e0 += 32) {
        const int e = e0 + lane;
        int mb = 0;
        if (e < p.groups) {
          int m = __ldg(p.masked_m + e);
          if (m < 0 || m > p.rows) {
            record_status(p.status, DG_ERR_DEVICE_DATA);
            m = m < 0 ? 0 : p.rows;
          }
          mb = (m + BM - 1) / BM;
          s_mblocks[e] = mb;
        }
        int v = mb * p.num_n_blocks, incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (e < p.groups) s_prefix[e] = running + incl - v;
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_prefix[p.groups] = running;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int units = num_units(p, SCHED, s_prefix);

  if (warp == 0) {
    // ============================================================ producer
    int it = 0;
    bool alive = true;
    for (int u = blockIdx.x; u < units && alive; u += gridDim.x) {
      Tile t = unit_to_tile(p, SCHED, u, s_prefix, s_mblocks);
      if constexpr (SCHED == kContiguous) {
        t.group = block_expert(p, t.m_blk, true);
        if (t.group < 0) continue;
      }
      const int a_row = t.m_blk * BM, b_row = t.n_blk * BN;
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1, s_abort, p.status)) { alive = false; break; }
        if (lane == 0) {
          const uint32_t sa = base + s * L::kStageBytes;
          mbar_arrive_expect_tx(full_bar(s), L::kStageBytes);
          tma_load_3d(sa, &tmap_a, full_bar(s), kb * BK, a_row, t.slab);
          tma_load_3d(sa + kABytes, &tmap_b, full_bar(s), kb * BK, b_row, t.group);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
    int it = 0, acc_it = 0;
    bool alive = true;
    for (int u = blockIdx.x; u < units && alive; u += gridDim.x) {
      Tile t = unit_to_tile(p, SCHED, u, s_prefix, s_mblocks);
      if constexpr (SCHED == kContiguous) {
        if (block_expert(p, t.m_blk, false) < 0) continue;
      }
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it, ++acc_it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int buf = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (!mbar_wait(tempty_bar(buf), aph ^ 1, s_abort, p.status)) { alive = false; break; }
        if (!mbar_wait(full_bar(s), ph, s_abort, p.status)) { alive = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sa = base + s * L::kStageBytes;
          const uint64_t adesc = smem_desc_k128_sw128(sa);
          const uint64_t bdesc = smem_desc_k128_sw128(sa + kABytes);
          const uint32_t d = tmem_base + buf * BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            // +32 bytes along K inside the swizzled 128-byte row = +2 in the
            // descriptor's 16-byte address field
            umma_f8(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
          umma_commit(tfull_bar(buf));
        }
        __syncwarp();
      }
    }
    // make sure every MMA issued above has completed before TMEM is freed
    // (bounded, and not cut short by the abort flag)
    if (lane == 0) umma_commit(drain_bar);
    __syncwarp();
    volatile int never = 0;
    mbar_wait(drain_bar, 0, &never, p.status);
  } else if (warp >= 4) {
    // ============================================================ promotion
    const int pw = warp - 4;           // 0..7
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31
    const int half = pw >> 2;          // column half of the tile
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const int nb_total = (p.n + 127) / 128;
    const int kg_total = p.num_k_blocks;
    int acc_it = 0;
    bool alive = true;
    for (int u = blockIdx.x; u < units && alive; u += gridDim.x) {
      Tile t = unit_to_tile(p, SCHED, u, s_prefix, s_mblocks);
      const int row = t.m_blk * BM + row_in_tile;
      bool row_ok;
      if constexpr (SCHED == kContiguous) {
        t.group = block_expert(p, t.m_blk, false);
        if (t.group < 0) continue;
        row_ok = row < p.rows && __ldg(p.m_indices + row) == t.group;
      } else if constexpr (SCHED == kMasked) {
        int m = __ldg(p.masked_m + t.slab);
        m = m < 0 ? 0 : (m > p.rows ? p.rows : m);
        row_ok = row < m;
      } else {
        row_ok = row < p.rows;
      }
      const int col0 = t.n_blk * BN + half * W;  // first column of this thread
      const int row_c = row < p.rows ? row : p.rows - 1;
      const float *sfa_ptr =
          p.sfa + static_cast<int64_t>(t.slab) * kg_total * p.ld_sfa + row_c;
      const int nb = min(col0, p.n - 1) / 128;
      const float *sfb_ptr =
          p.sfb + (static_cast<int64_t>(t.group) * nb_total + nb) * kg_total;

      float acc[W];
#pragma unroll
      for (int c = 0; c < W; ++c) acc[c] = 0.0f;

      float a_next = __ldg(sfa_ptr + static_cast<int64_t>(t.k_begin) * p.ld_sfa);
      float b_next = __ldg(sfb_ptr + t.k_begin);
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++acc_it) {
        const float a_cur = a_next, b_cur = b_next;
        if (kb + 1 < t.k_end) {
          a_next = __ldg(sfa_ptr + static_cast<int64_t>(kb + 1) * p.ld_sfa);
          b_next = __ldg(sfb_ptr + kb + 1);
        }
        const int buf = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (!mbar_wait(tfull_bar(buf), aph, s_abort, p.status)) { alive = false; break; }
        tc_fence_after();
        uint32_t r[W];
        tmem_ld<W>(tmem_base + t_lane + buf * BN + half * W, r);
        tmem_wait_ld();
        reg_barrier<W>(r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(buf));
        const float sc = a_cur * b_cur;
#pragma unroll
        for (int c = 0; c < W; ++c) acc[c] = fmaf(__uint_as_float(r[c]), sc, acc[c]);
      }
      if (!alive) break;

      // ---------------------------------------------------------- epilogue
      if (p.splits > 1) {
        if (*s_abort) break;
        // write this split's FP32 partial; the last arriving CTA reduces
        const int tile = u / p.splits;
        float *mine = p.ws + ((static_cast<int64_t>(tile) * p.splits + t.split) * BM +
                              row_in_tile) * BN + half * W;
#pragma unroll
        for (int c = 0; c < W; c += 4)
          __stcg(reinterpret_cast<float4 *>(mine + c),
                 make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"n"(kPromoThreads) : "memory");
        if (threadIdx.x == 4 * 32) {
          const uint32_t prev = atomicAdd(p.ws_ticket + tile, 1u);
          const int last = prev == static_cast<uint32_t>(p.splits - 1);
          if (last) p.ws_ticket[tile] = 0;  // ready for the next call
          *s_flag = last;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kPromoThreads) : "memory");
        if (!*s_flag) continue;
        __threadfence();
#pragma unroll
        for (int c = 0; c < W; ++c) acc[c] = 0.0f;
        for (int s = 0; s < p.splits; ++s) {
          const float *src = p.ws + ((static_cast<int64_t>(tile) * p.splits + s) * BM +
                                     row_in_tile) * BN + half * W;
#pragma unroll
          for (int c = 0; c < W; c += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + c));
            acc[c] += v.x; acc[c + 1] += v.y; acc[c + 2] += v.z; acc[c + 3] += v.w;
          }
        }
      }
      if (row_ok) {
        uint16_t *drow = p.d + (static_cast<int64_t>(t.slab) * p.rows + row) * p.n;
#pragma unroll
        for (int c = 0; c < W; c += 8) {
          if (col0 + c < p.n) {
            uint4 v;
            uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(acc[c + 2 * j], acc[c + 2 * j + 1]);
              w[j] = *reinterpret_cast<const uint32_t *>(&h);
            }
            *reinterpret_cast<uint4 *>(drow + col0 + c) = v;
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, L::kTmemCols);
}

// ------------------------------------------------------------------ host side
template <int BN, int STAGES>
constexpr int smem_bytes_for(int groups_extra) {
  return 1024 + STAGES * Layout<BN>::kStageBytes + 8 * (2 * STAGES + 5) + 16 +
         groups_extra;
}

struct Candidate {
  int bn;
  int stages;
};
constexpr Candidate kCandidates[] = {{128, 6}, {64, 8}, {32, 8}, {16, 8}};

template <int BN, int STAGES, int SCHED>
int launch_instance(const CUtensorMap &ta, const CUtensorMap &tb,
                    const GemmParams &p, int grid, int extra_smem,
                    cudaStream_t stream) {
  const int smem = smem_bytes_for<BN, STAGES>(extra_smem);
  auto kern = fp8_gemm_kernel<BN, STAGES, SCHED>;
  static int configured_smem[64] = {0};  // per device; grows only
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DG_ERR_CUDA;
  if (smem > configured_smem[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return DG_ERR_CUDA;
    configured_smem[dev] = smem;
  }
  kern<<<grid, kThreads, smem, stream>>>(ta, tb, p);
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

template <int SCHED>
int dispatch(int bn, const CUtensorMap &ta, const CUtensorMap &tb,
             const GemmParams &p, int grid, int extra, cudaStream_t st) {
  switch (bn) {
    case 128: return launch_instance<128, 6, SCHED>(ta, tb, p, grid, extra, st);
    case 64: return launch_instance<64, 8, SCHED>(ta, tb, p, grid, extra, st);
    case 32: return launch_instance<32, 8, SCHED>(ta, tb, p, grid, extra, st);
    case 16: return launch_instance<16, 8, SCHED>(ta, tb, p, grid, extra, st);
    default: return DG_ERR_INVALID_ARG;
  }
}

// 3-D tensor map over an E4M3 tensor [dim2][dim1][K] with a box of
// [1][box_rows][128] and the 128-byte swizzle.
int make_tmap(CUtensorMap *m, const void *ptr, int64_t k, int64_t rows,
              int64_t slabs, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return DG_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(k),
                                 static_cast<cuuint64_t>(k * rows)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

bool print_configs() {
  static const int v = [] {
    const char *e = getenv("DG_PRINT_CONFIGS");
    return (e && *e && *e != '0') ? 1 : 0;
  }();
  return v != 0;
}

// Estimated time (arbitrary units) of a config: waves x per-tile time, with
// per-tile time the larger of tensor time and operand-feed time per K block,
// and a floor from streaming every distinct byte once through HBM.
double estimate(int64_t m_blocks, int64_t n, int64_t k, int bn, int splits,
                int sms) {
  const int64_t n_blocks = (n + bn - 1) / bn;
  const int64_t units = m_blocks * n_blocks * splits;
  const int64_t waves = (units + sms - 1) / sms;
  const double kb = static_cast<double>(k / BK) / splits;
  // cycles per K block: MMA 128 x bn x 128 at ~8192 MAC/clk; operand feed
  // (16 KB + bn*128 B) at ~64 B/clk from L2; fixed ~120 cycles of latency.
  const double mma = 2.0 * bn;
  const double feed = (16384.0 + 128.0 * bn) / 64.0;
  const double per_tile = kb * std::max(mma, feed) + 400.0 + 4.0 * bn;
  double t = waves * per_tile;
  // HBM floor: B once + A once, at ~23 B/clk/SM aggregated over all SMs
  const double bytes = static_cast<double>(n) * k + m_blocks * 128.0 * k;
  t = std::max(t, bytes / (23.0 * sms));
  if (splits > 1) t += 600.0;  // reduction pass and its latency
  return t;
}

}  // namespace

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)num_sms;
  if (M <= 0 || M > 2 * BM) return 0;
  // largest possible split-K footprint: BN 16, up to 8 splits
  const int64_t m_blocks = (M + BM - 1) / BM;
  size_t best = 0;
  for (const Candidate &c : kCandidates) {
    const int64_t tiles = m_blocks * ((N + c.bn - 1) / c.bn);
    const size_t bytes = static_cast<size_t>(tiles) * 8 * BM * c.bn * 4 + tiles * 4 + 16;
    best = std::max(best, bytes);
  }
  (void)K;
  return (best + 255) & ~static_cast<size_t>(255);
}

int launch_fp8_gemm(int sched, const uint8_t *A, const uint8_t *B, GemmParams p,
                    cudaStream_t stream, int num_sms, size_t ws_bytes, void *ws) {
  const int64_t rows = p.rows, n = p.n, k = p.k;
  p.num_m_blocks = static_cast<int>((rows + BM - 1) / BM);
  p.num_k_blocks = static_cast<int>(k / BK);

  // ------------------------------------------------ choose BN (and splits)
  int bn = 128, splits = 1;
  double best = 1e300;
  const int64_t m_blocks_eff = sched == kMasked ? p.num_m_blocks * p.groups : p.num_m_blocks;
  const int64_t n_eff = sched == kDense ? n : n;  // B per expert
  for (const Candidate &c : kCandidates) {
    for (int s = 1; s <= 8; s *= 2) {
      if (s > 1 && (sched != kDense || ws == nullptr || p.num_m_blocks > 2)) break;
      if (s > p.num_k_blocks) break;
      const int64_t tiles = p.num_m_blocks * ((n + c.bn - 1) / c.bn);
      if (s > 1) {
        const size_t need = static_cast<size_t>(tiles) * s * BM * c.bn * 4 + tiles * 4;
        if (need > ws_bytes) break;
      }
      double e = estimate(m_blocks_eff, n_eff, k, c.bn, s, num_sms);
      if (sched == kMasked) e = estimate(m_blocks_eff, n, k, c.bn, s, num_sms);
      if (e < best * 0.97) {
        best = e;
        bn = c.bn;
        splits = s;
      }
    }
  }
  // Tuning / test overrides: DG_BLOCK_N forces the N tile, DG_SPLITS the K
  // split (dense only; needs enough workspace).
  if (const char *e = getenv("DG_BLOCK_N")) {
    const int v = atoi(e);
    for (const Candidate &c : kCandidates)
      if (c.bn == v) bn = v;
  }
  if (const char *e = getenv("DG_SPLITS")) {
    const int v = atoi(e);
    if (v >= 1) {
      const int64_t tiles = static_cast<int64_t>(p.num_m_blocks) * ((n + bn - 1) / bn);
      const size_t need = static_cast<size_t>(tiles) * v * BM * bn * 4 + tiles * 4;
      if (v > 1 && (sched != kDense || ws == nullptr || need > ws_bytes || v > p.num_k_blocks))
        return DG_ERR_WORKSPACE;
      splits = v;
    }
  }
  p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
  p.splits = splits;
  if (splits > 1) {
    const int64_t tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
    const size_t part = static_cast<size_t>(tiles) * splits * BM * bn * 4;
    p.ws = static_cast<float *>(ws);
    p.ws_ticket = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + part);
    if (cudaMemsetAsync(p.ws_ticket, 0, tiles * 4, stream) != cudaSuccess) return DG_ERR_CUDA;
  } else {
    p.ws = nullptr;
    p.ws_ticket = nullptr;
  }

  // ------------------------------------------------ tensor maps
  CUtensorMap ta, tb;
  const int64_t a_slabs = sched == kMasked ? p.groups : 1;
  int rc = make_tmap(&ta, A, k, rows, a_slabs, BM);
  if (rc) return rc;
  rc = make_tmap(&tb, B, k, n, sched == kDense ? 1 : p.groups, bn);
  if (rc) return rc;

  // ------------------------------------------------ grid
  int64_t units;
  int extra = 0;
  if (sched == kMasked) {
    units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks * p.groups;  // upper bound
    extra = 8 * (p.groups + 1);
  } else {
    units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks * splits;
  }
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
  if (print_configs()) {
    fprintf(stderr,
            "[dg] gemm sched=%d rows=%lld n=%lld k=%lld groups=%d: BN=%d splits=%d "
            "grid=%d units=%lld\n",
            sched, static_cast<long long>(rows), static_cast<long long>(n),
            static_cast<long long>(k), p.groups, bn, splits, grid,
            static_cast<long long>(units));
  }
  switch (sched) {
    case kDense: return dispatch<kDense>(bn, ta, tb, p, grid, extra, stream);
    case kContiguous: return dispatch<kContiguous>(bn, ta, tb, p, grid, extra, stream);
    case kMasked: return dispatch<kMasked>(bn, ta, tb, p, grid, extra, stream);
    default: return DG_ERR_INVALID_ARG;
  }
}

}  // namespace dg
