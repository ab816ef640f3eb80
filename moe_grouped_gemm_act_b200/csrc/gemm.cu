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
//   warp 0      TMA producer: one lane streams A [128 x 128] and B [BN x 128]
//               K blocks into a STAGES-deep shared-memory ring (128-byte
//               swizzle), and the block's 128 row scales alpha (one 512-byte
//               bulk copy from the MN-major scale array) into a separate ring
//               of kAlphaSlots slots, all completing on mbarriers.
//   warp 1      MMA issuer: allocates TMEM and, for each K block, issues 4
//               tcgen05.mma (kind::f8f6f4, M=128, N=BN, K=32) into one of NBUF
//               TMEM buffers (the first with accumulate off: a fresh partial
//               sum per block), then tcgen05.commit frees the smem stage and
//               publishes the buffer.  NBUF buffers let the tensor cores run
//               up to NBUF blocks ahead of the promotion.
//   warps 2-3   idle after set-up (warp 2 builds the masked prefix table);
//               warps 0-3 form the control warpgroup, whose registers the
//               promotion warpgroups take over for BN = 256.
//   warps 4-11  promotion: warp w reads TMEM lanes 32 (w mod 4) .. +31; warps
//               4-7 and 8-11 split the BN columns.  Each thread owns one row
//               and BN/2 columns: it pulls the block's partial sum with
//               tcgen05.ld, releases the buffer, and does acc += partial *
//               (alpha_row * beta) in FP32 registers.  After the last K block
//               it converts to BF16 and stores its row segment (valid rows).
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
constexpr int kControlWarps = 4;        // producer, MMA issuer, 2 helpers (one warpgroup)
constexpr int kPromoWarps = 8;          // two column halves x four lane quarters
constexpr int kPromoThreads = 32 * kPromoWarps;
constexpr int kThreads = 32 * (kControlWarps + kPromoWarps);
constexpr int kAlphaSlots = 16;         // alpha ring depth (>= STAGES + NBUF)
constexpr int kRasterGroupM = 16;       // M blocks per raster group (dense)
constexpr uint32_t kABytes = BM * BK;   // 16 KB per stage

template <int BN, int STAGES, int NBUF>
struct Layout {
  static constexpr uint32_t kBBytes = BN * BK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kAlphaOff = STAGES * kStageBytes;
  static constexpr uint32_t kBarOff = kAlphaOff + kAlphaSlots * BM * 4;
  // full[S] empty[S] afull[A] aempty[A] tfull[NBUF] tempty[NBUF] drain
  static constexpr uint32_t kNumBars = 2 * STAGES + 2 * kAlphaSlots + 2 * NBUF + 1;
  static constexpr uint32_t kMiscOff = kBarOff + 8 * kNumBars;
  static constexpr uint32_t kPrefixOff = kMiscOff + 16;
  static constexpr uint32_t kCols = BN * NBUF;
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64
                                      : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "TMEM holds 512 columns");
  static_assert(STAGES + NBUF <= kAlphaSlots, "alpha ring must cover the pipeline");
};

// ------------------------------------------------------------------ scheduler
struct Tile {
  int m_blk, n_blk, split;
  int slab;     // A / D slab (expert for masked, else 0)
  int group;    // B / beta group (expert, 0 for dense)
  int k_begin, k_end;  // K blocks of this unit
};

__device__ __forceinline__ int num_units(const GemmParams &p, int sched,
                                         const int *s_prefix) {
  if (sched == kMasked) return s_prefix[p.groups];
  return p.num_m_blocks * p.num_n_blocks * p.splits;
}

// Maps unit u to a tile.  The contiguous expert lookup is done separately.
__device__ __forceinline__ Tile unit_to_tile(const GemmParams &p, int sched,
                                             int u, const int *s_prefix,
                                             const int *s_mblocks) {
  Tile t;
  t.split = 0;
  t.slab = 0;
  t.group = 0;
  if (sched == kMasked) {
    // largest e with prefix[e] <= u; within an expert, the M blocks of one N
    // block are adjacent so that they share B in L2
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
  const int kb = p.num_k_blocks, s = p.splits;
  t.k_begin = (kb * t.split) / s;
  t.k_end = (kb * (t.split + 1)) / s;
  return t;
}

// Contiguous layout: the expert of a 128-row block, or -1 when the block holds
// only padding.  Whole warp; every lane returns the same value.  With `check`,
// a block mixing experts or holding an index >= groups records
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
  const unsigned any = __ballot_sync(0xffffffffu, first != 0x7FFFFFFF);
  if (!any) return -1;
  const int e = __shfl_sync(0xffffffffu, first, __ffs(any) - 1);
  if (check) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) bad |= (vals[i] >= 0 && vals[i] != e);
    bad |= (e >= p.groups);
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(p.status, DG_ERR_DEVICE_DATA);
  }
  return e < p.groups ? e : -1;
}

__device__ __forceinline__ int masked_rows(const GemmParams &p, int e) {
  const int m = __ldg(p.masked_m + e);
  return m < 0 ? 0 : (m > p.rows ? p.rows : m);
}

// ------------------------------------------------------------------ the kernel
template <int BN, int STAGES, int NBUF, int SCHED>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
  using L = Layout<BN, STAGES, NBUF>;
  constexpr int W = BN / 2;                 // columns per promotion thread
  // columns per TMEM load chunk: the whole slice up to 64; for BN = 256 the
  // 128 accumulators leave room for 16-column chunks under 168 registers
  constexpr int LW = W <= 64 ? W : 16;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(W % LW == 0 && (LW == 8 || LW == 16 || LW == 32 || LW == 64), "TMEM chunk");

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);

  const uint32_t bars = base + L::kBarOff;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto afull_bar = [&](int s) { return bars + 8u * (2 * STAGES + s); };
  auto aempty_bar = [&](int s) { return bars + 8u * (2 * STAGES + kAlphaSlots + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * STAGES + 2 * kAlphaSlots + b); };
  auto tempty_bar = [&](int b) {
    return bars + 8u * (2 * STAGES + 2 * kAlphaSlots + NBUF + b);
  };
  const uint32_t drain_bar = bars + 8u * (L::kNumBars - 1);
  const float *s_alpha = reinterpret_cast<const float *>(smem + L::kAlphaOff);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  int *s_flag = reinterpret_cast<int *>(smem + L::kMiscOff + 8);
  int *s_prefix = reinterpret_cast<int *>(smem + L::kPrefixOff);        // [groups + 1]
  int *s_mblocks = s_prefix + (SCHED == kMasked ? p.groups + 1 : 0);   // [groups]

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
    for (int s = 0; s < kAlphaSlots; ++s) {
      mbar_init(afull_bar(s), 1);
      mbar_init(aempty_bar(s), kPromoWarps);
    }
    for (int b = 0; b < NBUF; ++b) {
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
      // prefix[e] = sum_{e' < e} ceil(clamp(masked_m[e']) / 128) * n_blocks
      int running = 0;
      for (int e0 = 0; e0 < p.groups; e0 += 32) {
        const int e = e0 + lane;
        int mb = 0;
        if (e < p.groups) {
          const int m = __ldg(p.masked_m + e);
          if (m < 0 || m > p.rows) record_status(p.status, DG_ERR_DEVICE_DATA);
          mb = (masked_rows(p, e) + BM - 1) / BM;
          s_mblocks[e] = mb;
        }
        const int v = mb * p.num_n_blocks;
        int incl = v;
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
  const int kg_total = p.num_k_blocks;

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
      // alpha slice of this M block: rows a_row .. a_row+127 of the MN-major
      // array, clipped to the leading dimension (a multiple of 4 floats)
      const int64_t a_avail = p.ld_sfa - a_row;
      const uint32_t a_bytes = static_cast<uint32_t>(4 * (a_avail < BM ? a_avail : BM));
      const float *a_src = p.sfa + static_cast<int64_t>(t.slab) * kg_total * p.ld_sfa + a_row;
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int as = it % kAlphaSlots;
        const uint32_t aph = (it / kAlphaSlots) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1, s_abort, p.status)) { alive = false; break; }
        if (!mbar_wait(aempty_bar(as), aph ^ 1, s_abort, p.status)) { alive = false; break; }
        if (lane == 0) {
          const uint32_t sa = base + s * L::kStageBytes;
          mbar_arrive_expect_tx(full_bar(s), L::kStageBytes);
          tma_load_3d(sa, &tmap_a, full_bar(s), kb * BK, a_row, t.slab);
          tma_load_3d(sa + kABytes, &tmap_b, full_bar(s), kb * BK, b_row, t.group);
          mbar_arrive_expect_tx(afull_bar(as), a_bytes);
          bulk_load(base + L::kAlphaOff + as * (BM * 4), a_src + static_cast<int64_t>(kb) * p.ld_sfa,
                    a_bytes, afull_bar(as));
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
        const int buf = acc_it % NBUF;
        const uint32_t bph = (acc_it / NBUF) & 1;
        if (!mbar_wait(tempty_bar(buf), bph ^ 1, s_abort, p.status)) { alive = false; break; }
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
    // every MMA issued above must complete before TMEM is freed (bounded, and
    // not cut short by the abort flag)
    if (lane == 0) umma_commit(drain_bar);
    __syncwarp();
    volatile int never = 0;
    mbar_wait(drain_bar, 0, &never, p.status);
  } else if (warp >= kControlWarps) {
    // ============================================================ promotion
    const int pw = warp - kControlWarps;   // 0..7
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int half = pw >> 2;              // column half of the tile
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const int nb_total = (p.n + 127) / 128;
    int it = 0;
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
        row_ok = row < masked_rows(p, t.slab);
      } else {
        row_ok = row < p.rows;
      }
      const int col0 = t.n_blk * BN + half * W;  // first column of this thread
      // a thread's W columns (W divides 128 or equals 128) lie in one beta block
      const int nb = min(col0, p.n - 1) / 128;
      const float *sfb_ptr =
          p.sfb + (static_cast<int64_t>(t.group) * nb_total + nb) * kg_total;

      float acc[W];
#pragma unroll
      for (int c = 0; c < W; ++c) acc[c] = 0.0f;

      float b_next = __ldg(sfb_ptr + t.k_begin);
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        const float b_cur = b_next;
        if (kb + 1 < t.k_end) b_next = __ldg(sfb_ptr + kb + 1);
        const int as = it % kAlphaSlots;
        const int buf = it % NBUF;
        if (!mbar_wait(afull_bar(as), (it / kAlphaSlots) & 1, s_abort, p.status)) {
          alive = false;
          break;
        }
        const float sc = s_alpha[as * BM + row_in_tile] * b_cur;
        __syncwarp();
        if (lane == 0) mbar_arrive(aempty_bar(as));
        if (!mbar_wait(tfull_bar(buf), (it / NBUF) & 1, s_abort, p.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < W; c0 += LW) {
          uint32_t r[LW];
          tmem_ld<LW>(tmem_base + t_lane + buf * BN + half * W + c0, r);
          tmem_wait_ld();
          reg_barrier<LW>(r);
          if (c0 + LW == W) {
            // all of this buffer has been read: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(buf));
          }
#pragma unroll
          for (int c = 0; c < LW; ++c) acc[c0 + c] = fmaf(__uint_as_float(r[c]), sc, acc[c0 + c]);
        }
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
        if (threadIdx.x == kControlWarps * 32) {
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
struct Candidate {
  int bn, stages, nbuf;
};
// N tiles and their pipeline depths: 4-6 stages keep ~200 KB of operands in
// flight; NBUF fills the 512 TMEM columns (at most 8 buffers).
constexpr Candidate kCandidates[] = {
    {256, 4, 2}, {128, 6, 4}, {64, 8, 8}, {32, 8, 8}, {16, 8, 8}};

template <int BN, int STAGES, int NBUF>
constexpr int smem_bytes_for(int extra) {
  return 1024 + Layout<BN, STAGES, NBUF>::kPrefixOff + extra;
}

template <int BN, int STAGES, int NBUF, int SCHED>
int launch_instance(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p,
                    int grid, int extra_smem, cudaStream_t stream) {
  const int smem = smem_bytes_for<BN, STAGES, NBUF>(extra_smem);
  auto kern = fp8_gemm_kernel<BN, STAGES, NBUF, SCHED>;
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
int dispatch(int bn, const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p,
             int grid, int extra, cudaStream_t st) {
  switch (bn) {
    case 256: return launch_instance<256, 4, 2, SCHED>(ta, tb, p, grid, extra, st);
    case 128: return launch_instance<128, 6, 4, SCHED>(ta, tb, p, grid, extra, st);
    case 64: return launch_instance<64, 8, 8, SCHED>(ta, tb, p, grid, extra, st);
    case 32: return launch_instance<32, 8, 8, SCHED>(ta, tb, p, grid, extra, st);
    case 16: return launch_instance<16, 8, 8, SCHED>(ta, tb, p, grid, extra, st);
    default: return DG_ERR_INVALID_ARG;
  }
}

// 3-D tensor map over an E4M3 tensor [dim2][dim1][K] with a box of
// [1][box_rows][128] and the 128-byte swizzle.
int make_tmap(CUtensorMap *m, const void *ptr, int64_t k, int64_t rows, int64_t slabs,
              int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return DG_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(k * rows)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

bool print_configs() {
  const char *e = getenv("DG_PRINT_CONFIGS");
  return e && *e && *e != '0';
}

// Estimated time (SM cycles) of a config: waves x per-unit time, with per-unit
// time the larger of tensor time and operand-feed time per K block plus a
// fixed tile overhead, and a floor from streaming the distinct bytes once
// through HBM.
double estimate(int64_t m_blocks, int64_t n, int64_t k, int bn, int splits, int sms) {
  const int64_t n_blocks = (n + bn - 1) / bn;
  const int64_t units = m_blocks * n_blocks * splits;
  const int64_t waves = (units + sms - 1) / sms;
  const double kb = static_cast<double>(k / BK) / splits;
  const double mma = 2.0 * bn;                             // 128 x bn x 128 / 8192 per clk
  const double feed = (16384.0 + 128.0 * bn) / 96.0;       // smem fill rate from L2
  const double per_unit = kb * std::max(mma, feed) + 800.0 + 4.0 * bn;
  double t = waves * per_unit;
  const double bytes = static_cast<double>(n) * k + m_blocks * 128.0 * k;
  t = std::max(t, bytes / (23.0 * sms));                   // ~6.5 TB/s of HBM
  if (splits > 1) t += 800.0;                              // reduction pass
  return t;
}

size_t split_ws_bytes(int64_t tiles, int splits, int bn) {
  return static_cast<size_t>(tiles) * splits * BM * bn * 4 + tiles * 4;
}

struct Choice {
  int bn, splits;
};

// Tile width and K split for a launch.  Splitting K is considered for dense
// shapes of at most two M blocks, and only when the workspace can hold the
// split's FP32 partials (`ws_bytes`).
Choice choose_config(int sched, int64_t rows, int64_t n, int64_t k, int groups, int num_sms,
                     size_t ws_bytes) {
  const int64_t m_blocks = (rows + BM - 1) / BM;
  const int64_t k_blocks = k / BK;
  const int64_t m_blocks_eff = sched == kMasked ? m_blocks * groups : m_blocks;
  Choice c{128, 1};
  double best = 1e300;
  for (const Candidate &cand : kCandidates) {
    for (int s = 1; s <= 8; s *= 2) {
      if (s > 1 && (sched != kDense || m_blocks > 2)) break;
      if (s > k_blocks) break;
      const int64_t tiles = m_blocks * ((n + cand.bn - 1) / cand.bn);
      if (s > 1 && split_ws_bytes(tiles, s, cand.bn) > ws_bytes) break;
      const double e = estimate(m_blocks_eff, n, k, cand.bn, s, num_sms);
      if (e < best * 0.97) {
        best = e;
        c = {cand.bn, s};
      }
    }
  }
  return c;
}

}  // namespace

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  // the split the heuristic picks when the workspace is not a constraint
  const Choice c = choose_config(kDense, M, N, K, 1, num_sms, ~static_cast<size_t>(0));
  if (c.splits <= 1) return 0;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + c.bn - 1) / c.bn);
  return (split_ws_bytes(tiles, c.splits, c.bn) + 255) & ~static_cast<size_t>(255);
}

int launch_fp8_gemm(int sched, const uint8_t *A, const uint8_t *B, GemmParams p,
                    cudaStream_t stream, int num_sms, size_t ws_bytes, void *ws) {
  const int64_t rows = p.rows, n = p.n, k = p.k;
  p.num_m_blocks = static_cast<int>((rows + BM - 1) / BM);
  p.num_k_blocks = static_cast<int>(k / BK);
  if (ws == nullptr) ws_bytes = 0;
  const int64_t m_blocks_eff =
      sched == kMasked ? static_cast<int64_t>(p.num_m_blocks) * p.groups : p.num_m_blocks;

  // ------------------------------------------------ choose BN (and splits)
  const Choice choice = choose_config(sched, rows, n, k, p.groups, num_sms, ws_bytes);
  int bn = choice.bn, splits = choice.splits;
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
      if (v > 1 && (sched != kDense || ws == nullptr || split_ws_bytes(tiles, v, bn) > ws_bytes ||
                    v > p.num_k_blocks))
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
  int rc = make_tmap(&ta, A, k, rows, sched == kMasked ? p.groups : 1, BM);
  if (rc) return rc;
  rc = make_tmap(&tb, B, k, n, sched == kDense ? 1 : p.groups, bn);
  if (rc) return rc;

  // ------------------------------------------------ grid
  int64_t units;
  int extra = 0;
  if (sched == kMasked) {
    units = m_blocks_eff * p.num_n_blocks;  // upper bound; actual from masked_m
    extra = 8 * (p.groups + 1);
  } else {
    units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks * splits;
  }
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
  if (print_configs()) {
    fprintf(stderr,
            "[dg] gemm sched=%d rows=%lld n=%lld k=%lld groups=%d: BN=%d splits=%d grid=%d "
            "units=%lld\n",
            sched, static_cast<long long>(rows), static_cast<long long>(n),
            static_cast<long long>(k), p.groups, bn, splits, grid, static_cast<long long>(units));
  }
  switch (sched) {
    case kDense: return dispatch<kDense>(bn, ta, tb, p, grid, extra, stream);
    case kContiguous: return dispatch<kContiguous>(bn, ta, tb, p, grid, extra, stream);
    case kMasked: return dispatch<kMasked>(bn, ta, tb, p, grid, extra, stream);
    default: return DG_ERR_INVALID_ARG;
  }
}

}  // namespace dg
