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
//               swizzle), completing on mbarriers.
//   warp 1      MMA issuer: allocates TMEM and, for each K block, issues 4
//               tcgen05.mma (kind::f8f6f4, M=128, N=BN, K=32) into one of NBUF
//               TMEM buffers (the first with accumulate off: a fresh partial
//               sum per block), then tcgen05.commit frees the smem stage and
//               publishes the buffer.  NBUF buffers let the tensor cores run
//               up to NBUF blocks ahead of the promotion.
//   warps 2-3   idle after set-up (warp 2 builds the masked or k-grouped
//               prefix table);
//               warps 0-3 form the control warpgroup, whose registers the
//               promotion warpgroups take over for BN = 256.
//   warps 4-11  promotion: warp w reads TMEM lanes 32 (w mod 4) .. +31; warps
//               4-7 and 8-11 split the BN columns.  Each thread owns one row
//               and BN/2 columns: it pulls the block's partial sum with
//               tcgen05.ld, releases the buffer, and does acc += partial *
//               (alpha_row * beta) in FP32 registers, two columns per packed
//               f32x2 FMA.  Its row scale alpha is loaded into registers two
//               K blocks ahead.  After the last K block it converts to BF16
//               and stores its row segment (valid rows).
//
// The kernel is persistent (one CTA per SM).  All roles walk the same tile
// sequence produced by a scheduler that knows the layouts:
//   dense       tiles of D in an M-grouped raster (L2 reuse of B);
//   contiguous  as dense over M_total, the expert of each 128-row block read
//               from the per-row index; blocks holding only padding skipped;
//   masked      per expert g, ceil(masked_m[g] / 128) row blocks x N blocks,
//               counts read on the device (launch shape independent of them);
//   k-grouped   the weight gradient ("DeepGEMM architecture deep dive",
//               section 3, the grouped GEMM table): per group, a dense raster
//               over its own K segment (sizes read on the device); B's scales
//               are per column, so the producer also copies each block's
//               slice of them into a shared-memory ring and the promotion
//               scales per element; the output is FP32 D[g] = C[g] + ....
// Dense small-M shapes split K (units = tile x split, one unit per CTA): the
// splits of a tile form one thread-block cluster, leave their FP32 partials
// in shared memory and each reduces a share over the cluster's distributed
// shared memory, summing splits 0, 1, ... in order.  When those clusters do
// not fit one wave, and for the tiles of a last partial wave of larger dense
// shapes, the partials go through a workspace instead (cooperative launch,
// one arrival counter per tile, the same summation order).
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
#include "quant_math.cuh"

namespace dg {

namespace {

constexpr int BM = 128;                 // rows per tile (one UMMA M)
constexpr int BK = 128;                 // K per block = one scale group
constexpr int kControlWarps = 4;        // producer, MMA issuer, 2 helpers (one warpgroup)
constexpr int kPromoWarps = 8;          // two column halves x four lane quarters
constexpr int kPromoThreads = 32 * kPromoWarps;
constexpr int kThreads = 32 * (kControlWarps + kPromoWarps);
// Register split of the 256-wide tile: the block is launched with 168
// registers per thread (65536 / 384, in steps of 8); the control warpgroup
// gives up most of them so that each promotion thread can hold its 128
// accumulators and a 64-column TMEM chunk.  Either split uses exactly the
// launch allocation (40 x 128 + 232 x 256 = 56 x 128 + 224 x 256 = 168 x 384);
// per schedule, the one with which ptxas spills least (the 2-CTA form:
// 80 / 124 bytes of spill stores / loads with 40 / 232, 20 / 48 with 56 / 224,
// 96 / 128 with fewer promotion registers; 28 % faster with 56 / 224).
constexpr int kLaunchRegs = 168;
__host__ __device__ constexpr bool wide_control(int sched) {
  return sched == kMasked || sched == kDenseCluster || is_ue8m0(sched) || sched == kDensePair;
}
__host__ __device__ constexpr int ctrl_regs(int sched) { return wide_control(sched) ? 56 : 40; }
__host__ __device__ constexpr int promo_regs(int sched) { return wide_control(sched) ? 224 : 232; }
static_assert(ctrl_regs(kDense) * 32 * kControlWarps + promo_regs(kDense) * kPromoThreads <=
                  kLaunchRegs * kThreads,
              "register split exceeds the launch allocation");
static_assert(ctrl_regs(kMasked) * 32 * kControlWarps + promo_regs(kMasked) * kPromoThreads <=
                  kLaunchRegs * kThreads,
              "register split exceeds the launch allocation");
// Whether an instance runs with the warpgroup register split: the 256-wide
// tiles (except contiguous: with the split, ptxas spills in its promotion
// loop, measured 40 % slower) and the wider non-power-of-two tiles of the
// cluster split.
__host__ __device__ constexpr int gcd_c(int a, int b) { return b == 0 ? a : gcd_c(b, a % b); }
__host__ __device__ constexpr bool uses_reg_split(int bn, int sched) {
  return (bn == 256 && sched != kContiguous) || (bn > 128 && sched == kDenseCluster);
}
constexpr int kRasterGroupM = 16;       // M blocks per raster group (dense)
constexpr int kCAhead = 8;              // K blocks between the C prefetch and the tile's end
constexpr uint32_t kABytes = BM * BK;   // 16 KB per stage
constexpr int kClusterNoFit = 1;        // launch_instance: clusters do not fit one wave
constexpr int kMaxClusterSplits = 8;    // K splits reduced inside one (portable) cluster
constexpr uint32_t kStoreBoxCols = 64;  // BF16 columns per TMA store box (128 bytes)

// How a schedule's epilogue stages the output tile in shared memory: 0 not
// at all, 1 the BF16 tile, 2 the FP32 tile (D = C + A B^T adds C as it
// leaves).
__host__ __device__ constexpr int staged_epilogue(int sched) {
  return sched == kDenseAcc ? 2 : (sched == kDense || sched == kMasked) ? 1 : 0;
}

// The staging kind an instance uses (every schedule, including the UE8M0
// and quantizing forms): the UE8M0 forms stage the BF16 tile 64 columns at a
// time (kind 3), which leaves room for a fourth stage beside their per-stage
// scale-factor areas.
__host__ __device__ constexpr int instance_staging(int sched) {
  return sched == kDenseQuant ? 0 : is_ue8m0(sched) ? 3 : staged_epilogue(base_sched(sched));
}

// Scale-factor bytes per stage of the UE8M0 schedules: the K block's packed
// word (four K groups) of each of the tile's 128 rows of A and 256 rows of
// B, arranged as tcgen05.cp's 32-row x 16-byte sources: row r of a source
// holds the words of tile rows r, r + 32, r + 64, r + 96.
constexpr uint32_t kSfABytes = 512;
constexpr uint32_t kSfStageBytes = kSfABytes + 1024;
// TMEM columns of the scale factors: two slots (consecutive K blocks) of 4
// (A) + 8 (B) columns, 16 apart.
constexpr uint32_t kSfSlotCols = 16;

template <int BN, int STAGES, int NBUF, int STAGED, bool KG = false, bool UE = false,
          bool PAIR = false>
struct Layout {
  // the 2-CTA form keeps half of the B tile (BN / 2 rows) in each CTA
  static constexpr uint32_t kBBytes = (PAIR ? BN / 2 : BN) * BK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  // With STAGED, staging of the output for coalesced stores: 128 rows x
  // kOutCols BF16 (kind 1: a 256-wide tile goes out in two column halves) or
  // FP32 (kind 2: 64-column phases), then one byte per row saying whether it
  // is stored
  static constexpr uint32_t kOutCols =
      STAGED >= 2 ? (BN < 64 ? BN : 64) : (BN < 128 ? BN : 128);
  static constexpr uint32_t kOutElem = STAGED == 2 ? 4 : 2;
  static constexpr uint32_t kOutOff = STAGES * kStageBytes;
  static constexpr uint32_t kRowOkOff = kOutOff + (STAGED ? BM * kOutCols * kOutElem : 0);
  static constexpr uint32_t kBarOff = kRowOkOff + (STAGED ? BM : 0);
  // full[S] empty[S] tfull[NBUF] tempty[NBUF] drain epi staged free
  static constexpr uint32_t kNumBars = 2 * STAGES + 2 * NBUF + 4;
  static constexpr uint32_t kMiscOff = kBarOff + 8 * kNumBars;
  static constexpr uint32_t kPrefixOff = kMiscOff + 16;
  // k-grouped: a ring of per-column B scale slices, one per K block in
  // flight (STAGES in the shared-memory stages plus NBUF in the TMEM
  // buffers), so the producer never refills a slot the promotion may still
  // read; then the per-schedule tables (masked / k-grouped prefix sums)
  static constexpr int kBetaSlots = KG ? STAGES + NBUF : 0;
  static constexpr uint32_t kBetaOff = (kPrefixOff + 15u) & ~15u;
  static constexpr uint32_t kBetaBytes = static_cast<uint32_t>(kBetaSlots) * BN * 4u;
  // UE8M0 schedules: a scale-factor area per stage (128-byte aligned)
  static constexpr uint32_t kSfOff = (kBetaOff + kBetaBytes + 127u) & ~127u;
  static constexpr uint32_t kSfBytes = UE ? STAGES * kSfStageBytes : 0u;
  static constexpr uint32_t kTableOff = kSfOff + kSfBytes;
  static_assert(!UE || BN == 256, "the UE8M0 scale-factor layout is laid out for 256-wide tiles");
  // accumulator buffers (a non-power-of-two width starts each buffer on a
  // power-of-two column), then (UE8M0) the scale-factor slots
  static constexpr uint32_t kBufCols =
      (BN & (BN - 1)) == 0 ? BN : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr uint32_t kCols = kBufCols * NBUF + (UE ? 2 * kSfSlotCols : 0);
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64
                                      : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "TMEM holds 512 columns");
};

// ------------------------------------------------------------------ scheduler
struct Tile {
  int m_blk, n_blk;
  int tile;           // linear tile index (dense / contiguous)
  int split, nsplit;  // this unit's K split of the tile's nsplit
  int slab;     // A / D slab (expert for masked, else 0)
  int group;    // B / beta group (expert, 0 for dense)
  int k_begin, k_end;  // K blocks of this unit
};

__device__ __forceinline__ int num_units(const GemmParams &p, int sched,
                                         const int *s_prefix) {
  if (sched == kMasked) return s_prefix[p.groups];
  if (sched == kKGrouped) return p.groups * p.num_m_blocks * p.num_n_blocks;
  return p.full_tiles + (p.num_m_blocks * p.num_n_blocks - p.full_tiles) * p.splits;
}

// Maps unit u to a tile.  The contiguous expert lookup is done separately.
// Dense and contiguous: units 0 .. full_tiles-1 are whole tiles; each later
// tile is `splits` consecutive units (K ranges), so a split tile's units fall
// on distinct CTAs of the last wave.
__device__ __forceinline__ Tile unit_to_tile(const GemmParams &p, int sched,
                                             int u, const int *s_prefix,
                                             const int *s_mblocks) {
  Tile t;
  t.tile = 0;
  t.split = 0;
  t.nsplit = 1;
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
    int tile = u;
    if (sched == kKGrouped) {
      // groups one after the other, each rastered like a dense GEMM
      const int per_group = p.num_m_blocks * p.num_n_blocks;
      t.group = u / per_group;
      tile = u - t.group * per_group;
    } else if (u >= p.full_tiles) {
      const int v = u - p.full_tiles;
      tile = p.full_tiles + v / p.splits;
      t.split = v - (tile - p.full_tiles) * p.splits;
      t.nsplit = p.splits;
    }
    t.tile = tile;
    const int span = kRasterGroupM * p.num_n_blocks;
    const int grp = tile / span;
    const int first_m = grp * kRasterGroupM;
    const int gm = min(kRasterGroupM, p.num_m_blocks - first_m);
    const int r = tile - grp * span;
    t.m_blk = first_m + r % gm;
    t.n_blk = r / gm;
  }
  if (sched == kKGrouped) {
    // the group's K blocks (prefix sums of the group sizes, in K blocks)
    t.k_begin = s_prefix[t.group];
    t.k_end = s_prefix[t.group + 1];
    return t;
  }
  const int kb = p.num_k_blocks, s = t.nsplit;
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
template <int BN, int STAGES, int NBUF, int SCHED, int LAYOUT = kLayoutNT>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_d,
                const GemmParams p) {
  // dense and masked tiles leave through shared memory (coalesced row
  // stores); contiguous tiles store each thread's row segment directly
  // (measured 1 % faster for them)
  // the UE8M0 schedules walk the tiles of their base schedule
  constexpr bool kUE = is_ue8m0(SCHED);
  constexpr int S = base_sched(SCHED);
  static_assert(!kUE || NBUF == 1, "the UE8M0 schedules keep one accumulator per tile");
  // operands stored with K outermost (T of A, N of B) are MN-major tiles in
  // shared memory: K rows of 128 values, B in BN / 128 such columns
  constexpr bool kAmn = a_mn_major(LAYOUT);
  constexpr bool kBmn = b_mn_major(LAYOUT);
  static_assert(LAYOUT == kLayoutNT || ((S == kDense || S == kDenseCluster || S == kKGrouped) &&
                                         !kUE && (!kBmn || BN % 128 == 0)),
                "transposed layouts serve the dense and k-grouped schedules");
  // the quantizing epilogue writes each thread's row group itself
  constexpr bool kQ = SCHED == kDenseQuant;
  constexpr int kStaged = instance_staging(SCHED);
  constexpr bool kDenseLike =
      (S == kDense || S == kDenseAcc) && !kUE && !kQ && SCHED != kDensePair;
  static_assert(!kQ || BN == 256, "the quantizing epilogue needs whole 128-column groups");
  constexpr bool kKG = S == kKGrouped;
  // 2-CTA form: the cluster's two CTAs compute one 256-row tile
  constexpr bool kPair = SCHED == kDensePair;
  constexpr int TM = kPair ? 2 * BM : BM;   // rows per tile
  // dense tile schedules: B's first stages can be asked into L2 at entry
  constexpr bool kPrefetchB = S == kDense || S == kDenseCluster || S == kDenseAcc;
  // 128- and 256-wide BF16 tiles leave by TMA stores of the staged tile:
  // dense tiles always (rows and columns past D are clipped by the tensor
  // map), UE8M0 masked tiles whose 128 rows are all valid.  (The FP32-scale
  // masked instance keeps its row stores: with both paths in it, ptxas
  // spills and it ran 25 % slower.)
  constexpr bool kTmaStore =
      (S == kDense || (S == kMasked && kUE)) && (kStaged == 1 || kStaged == 3) && BN >= 128;
  // dense TMA-stored tiles hand the stores to warp 2: the promotion warps
  // write their columns into the staging tile and go on to the next tile;
  // warp 2 issues each staging use's TMA store and frees the tile once the
  // store has read it.  Warps writing one staging use: the half that owns it
  // (256 wide: two uses per tile) or both halves (128 wide: one use).
  constexpr bool kStoreWarp = kTmaStore && S == kDense && !kUE && !kPair;
  constexpr int kStoreUses = BN > 128 ? 2 : 1;
  constexpr int kStoreWriters = kStoreUses == 2 ? kPromoWarps / 2 : kPromoWarps;
  static_assert(!kPair || (BN == 256 && LAYOUT == kLayoutNT), "the 2-CTA form: NT, 256 wide");
  using L = Layout<BN, STAGES, NBUF, kStaged, kKG, kUE, kPair>;
  constexpr int W = BN / 2;                 // columns per promotion thread
  // the wide tiles run with the warpgroup register split (promo_regs per
  // promotion thread), the others fit the launch allocation as they are
  constexpr bool kRegSplit = uses_reg_split(BN, S);
  // columns per TMEM load chunk: the whole slice up to 64 (one wait per
  // chunk; the buffer is handed back after the last chunk's wait, so the
  // fewer chunks, the sooner the MMA warp can reuse it); 16 for a 256-wide
  // tile without the register split (128 accumulators under 168 registers).
  // Non-power-of-two tiles: the largest of 64 / 32 / 16 dividing the slice
  // under the split, else 16.  A thread's first column is a multiple of W, so
  // the 128-column boundaries of B's scale blocks fall on multiples of
  // gcd(W, 128) within its slice, and a chunk never straddles one.
  constexpr bool kPow2 = (BN & (BN - 1)) == 0;
  constexpr int LW = kPow2 ? (W <= 64 ? W : kRegSplit ? 64 : 16)
                           : kRegSplit ? (W % 64 == 0 ? 64 : W % 32 == 0 ? 32 : 16) : 16;
  // a thread's W columns may span two 128-column blocks of B's scales
  // (non-power-of-two tiles only)
  constexpr bool kStraddle = !kPow2;
  static_assert(kPow2 || (S == kDenseCluster && BN % 32 == 0 && !kUE && LAYOUT == kLayoutNT),
                "non-power-of-two tiles serve the NT cluster split, 32-column multiples");
  static_assert(kPow2 || gcd_c(W, 128) % LW == 0, "a TMEM chunk within one scale block");
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
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * STAGES + NBUF + b); };
  const uint32_t drain_bar = bars + 8u * (2 * STAGES + 2 * NBUF);
  // synchronises the promotion threads in the epilogue (bounded, unlike a
  // named barrier, so that an aborting warp cannot strand the others)
  const uint32_t epi_bar = drain_bar + 8u;
  // TMA-stored tiles: a staging use has been written (by its writer warps),
  // and a use's TMA store has finished reading the staging tile
  const uint32_t staged_bar = epi_bar + 8u;
  const uint32_t free_bar = epi_bar + 16u;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  int *s_flag = reinterpret_cast<int *>(smem + L::kMiscOff + 8);
  int *s_prefix = reinterpret_cast<int *>(smem + L::kTableOff);         // [groups + 1]
  int *s_mblocks = s_prefix + (S == kMasked ? p.groups + 1 : 0);   // [groups]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 2-CTA form: rank 0 issues the pair's MMAs; units are per cluster
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const int u_first = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int u_stride = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // ---------------------------------------------------------------- setup
  // the next kernel of the stream may begin its own set-up as our CTAs leave
  grid_launch_dependents();
  if constexpr (kPrefetchB) {
    // B's boxes of this CTA's first stages are asked into L2 before the
    // set-up, so that HBM is busy while the barriers and TMEM are prepared
    // (a decode-sized launch otherwise spends microseconds before its first
    // bytes).  Same coordinates as the producer's loads.  A prefetch only
    // fills L2, which the previous kernel's writes also go through, so it
    // may precede the dependency wait; dense tiles only (their schedule
    // needs no device data).
    if (warp == 3 && lane < STAGES && u_first < num_units(p, S, nullptr)) {
      const Tile t = unit_to_tile(p, S, u_first, nullptr, nullptr);
      const int kb = t.k_begin + lane;
      const int b_row = t.n_blk * BN + (kPair ? static_cast<int>(rank) * (BN / 2) : 0);
      if (kb < t.k_end) {
        if constexpr (kBmn) {
#pragma unroll
          for (int j = 0; j < BN / 128; ++j) tma_prefetch_3d(&tmap_b, b_row + 128 * j, kb * BK, 0);
        } else {
          tma_prefetch_3d(&tmap_b, kb * BK, b_row, 0);
        }
      }
    }
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    for (int s = 0; s < STAGES; ++s) {
      // UE8M0: the producer's arrival with the byte count, plus one arrival
      // per producer lane when its scale-factor copies have landed
      mbar_init(full_bar(s), kUE ? 33 : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(tfull_bar(b), 1);
      // 2-CTA form: the promotion warps of both CTAs hand rank 0's MMA warp
      // the buffer
      mbar_init(tempty_bar(b), kPair ? 2 * kPromoWarps : kPromoWarps);
    }
    mbar_init(drain_bar, 1);
    mbar_init(epi_bar, kPromoWarps);
    mbar_init(staged_bar, kStoreWriters);
    mbar_init(free_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(s_tmem), L::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(s_tmem), L::kTmemCols);
      tmem_relinquish();
    }
  }
  // nothing above touched global memory; from here on the previous kernel's
  // results (A, the scales, the index arrays) are visible
  grid_dependency_wait();
  if constexpr (S == kMasked) {
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
  if constexpr (kKG) {
    if (warp == 2) {
      // prefix[g] = K blocks of groups 0 .. g-1.  A size that is negative or
      // off the 128 grid, or sizes that do not add up to K, are recorded as
      // DG_ERR_DEVICE_DATA; every prefix is clamped to [0, K/128] (each lane
      // adds at most K/128, the running sum stops at K/128 + 1), so no group
      // reads past the operands or their scales.
      const int kb_all = p.num_k_blocks;
      int running = 0;
      for (int g0 = 0; g0 < p.groups; g0 += 32) {
        const int g = g0 + lane;
        int nb = 0;
        if (g < p.groups) {
          const int ks = __ldg(p.k_sizes + g);
          if (ks < 0 || ks % BK != 0) {
            record_status(p.status, DG_ERR_DEVICE_DATA);
          } else {
            nb = min(ks / BK, kb_all);
          }
        }
        int incl = nb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (g < p.groups) s_prefix[g] = min(running + incl - nb, kb_all);
        running = min(running + __shfl_sync(0xffffffffu, incl, 31), kb_all + 1);
      }
      if (lane == 0) {
        if (running != kb_all) record_status(p.status, DG_ERR_DEVICE_DATA);
        s_prefix[p.groups] = min(running, kb_all);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int units = num_units(p, S, s_prefix);
  const int kg_total = p.num_k_blocks;

  if (warp < kControlWarps) {
  // the control warpgroup (all four warps) hands its spare registers over
  if constexpr (kRegSplit) setmaxnreg_dec<ctrl_regs(SCHED)>();
  if (warp == 0) {
    // ============================================================ producer
    // bytes per stage: the A box (128 rows, or 64 when M <= 64: the MMA then
    // reads stale rows 64-127, which only reach output rows that are never
    // stored) and the B box
    const uint32_t stage_tx = static_cast<uint32_t>(p.a_box_rows) * BK + L::kBBytes;
    // test hook (GemmParams::starve_it): nothing completes the left-out
    // stage's `full` barrier, so the MMA warp's bounded wait on it runs out,
    // which exercises the abort path without faulting anything
    const int starve_it = blockIdx.x == 0 ? p.starve_it : -1;
    int it = 0;
    bool alive = true;
    for (int u = u_first; u < units && alive; u += u_stride) {
      Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
      if constexpr (S == kContiguous) {
        t.group = block_expert(p, t.m_blk, true);
        if (t.group < 0) continue;
      }
      const int a_row = t.m_blk * TM + static_cast<int>(rank) * BM;
      const int b_row = t.n_blk * BN + (kPair ? static_cast<int>(rank) * (BN / 2) : 0);
      // D = C + A B^T: the epilogue's C rows are asked into L2 kCAhead K
      // blocks before the tile's last one -- late enough that the operand
      // stream of a long K does not evict them first, early enough to cover
      // the DRAM latency the epilogue would otherwise wait on
      const int c_kb = (S == kDenseAcc && t.split == 0) ? max(t.k_begin, t.k_end - kCAhead)
                                                            : -1;
      // k-grouped: the tile's slice of B's column scales for each K block
      // (N % 8 == 0, so a multiple of 32 bytes; 16-byte aligned because the
      // scale rows are and the tile starts on a 16-column boundary)
      const int b_col0 = t.n_blk * BN;
      const uint32_t beta_bytes = kKG ? static_cast<uint32_t>(min(BN, p.n - b_col0)) * 4u : 0u;
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        if constexpr (S == kDenseAcc) {
          if (kb == c_kb) {
            const int col0 = t.n_blk * BN;
            const uint32_t bytes = static_cast<uint32_t>(min(BN, p.n - col0)) * 4u;
            const int valid = min(BM, p.rows - a_row);
            for (int r = lane; r < valid; r += 32)
              prefetch_l2_bulk(p.c + static_cast<int64_t>(a_row + r) * p.n + col0, bytes);
          }
        }
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1, s_abort, p.status)) { alive = false; break; }
        if (kPair && lane == 0 && it != starve_it) {
          // 2-CTA form: both CTAs' boxes complete on rank 0's `full`
          // barrier, which rank 0 arms for the pair's bytes
          const uint32_t sa = base + s * L::kStageBytes;
          const uint32_t fb = mapa_shared(full_bar(s), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * stage_tx);
          tma_load_3d_pair(sa, &tmap_a, fb, kb * BK, a_row, t.slab);
          tma_load_3d_pair(sa + kABytes, &tmap_b, fb, kb * BK, b_row, t.group);
        } else if (lane == 0 && it != starve_it) {
          const uint32_t sa = base + s * L::kStageBytes;
          // (the k-grouped form's B is one [N][K] tensor for all groups)
          const int b_slab = kKG ? 0 : t.group;
          mbar_arrive_expect_tx(full_bar(s), stage_tx + beta_bytes);
          if constexpr (kAmn) {
            tma_load_3d(sa, &tmap_a, full_bar(s), a_row, kb * BK, t.slab);
          } else {
            tma_load_3d(sa, &tmap_a, full_bar(s), kb * BK, a_row, t.slab);
          }
          if constexpr (kBmn) {
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tma_load_3d(sa + kABytes + j * (BK * 128), &tmap_b, full_bar(s), b_row + 128 * j,
                          kb * BK, b_slab);
          } else {
            tma_load_3d(sa + kABytes, &tmap_b, full_bar(s), kb * BK, b_row, b_slab);
          }
          if constexpr (kKG) {
            bulk_load(base + L::kBetaOff + static_cast<uint32_t>(it % L::kBetaSlots) * (BN * 4u),
                      p.sfb + static_cast<int64_t>(kb) * p.ld_sfb + b_col0, beta_bytes,
                      full_bar(s));
          }
        }
        if constexpr (kUE) {
          // The K block's packed scale words (four K groups each) of the
          // tile's rows of A and B, one 4-byte cp.async per word, placed as
          // tcgen05.cp's sources (lane l fills source row l); rows past the
          // operands take the last row's word (their outputs are not
          // stored).  Each lane then arrives on the stage's barrier once its
          // copies have landed.
          if (it != starve_it) {
            const uint32_t sf = base + L::kSfOff + static_cast<uint32_t>(s) * kSfStageBytes +
                                static_cast<uint32_t>(lane) * 16u;
            const int kwords = (kg_total + 3) / 4;
            const int32_t *wa = reinterpret_cast<const int32_t *>(p.sfa) +
                                (static_cast<int64_t>(t.slab) * kwords + kb / 4) * p.ld_sfa;
            const int32_t *wb = reinterpret_cast<const int32_t *>(p.sfb) +
                                (static_cast<int64_t>(t.group) * kwords + kb / 4) * p.ld_sfb;
#pragma unroll
            for (int m1 = 0; m1 < 4; ++m1)
              cp_async_4(sf + 4u * m1, wa + min(a_row + lane + 32 * m1, p.rows - 1));
#pragma unroll
            for (int n1 = 0; n1 < 8; ++n1)
              cp_async_4(sf + kSfABytes + 512u * (n1 >> 2) + 4u * (n1 & 3),
                         wb + min(b_row + lane + 32 * n1, p.n - 1));
            cp_async_arrive_noinc(full_bar(s));
          }
        }
        __syncwarp();
      }
    }
    // No copy may still be writing this CTA's shared memory when it exits:
    // wait (bounded, and not cut short by the abort flag) for the `full`
    // barrier of each of the last STAGES iterations armed above.  Earlier
    // iterations were consumed by the MMA warp, so their copies landed.
    // (2-CTA form: rank 0's barriers count both CTAs' bytes, and rank 1
    // leaves only after rank 0 at the teardown's cluster barrier.)
    volatile int never = 0;
    if (!kPair || rank == 0)
      for (int i = max(0, it - STAGES); i < it; ++i)
        if (i != starve_it) mbar_wait(full_bar(i % STAGES), (i / STAGES) & 1, &never, p.status);
  } else if (warp == 1) {
   if constexpr (kPair) {
    // (2-CTA form: rank 1's MMA warp has no loop; rank 0 issues the
    // pair's MMAs)
    if (rank == 0) {
      // ========================================= 2-CTA form, rank 0: MMAs
      // One cta_group::2 MMA of 256 x BN x 32 covers both CTAs' rows; its
      // completion frees both CTAs' stages and publishes both CTAs' TMEM
      // buffers (multicast commits).
      constexpr uint32_t idesc = idesc_e4m3_f32(2 * BM, BN);
      int it = 0, acc_it = 0;
      bool alive = true;
      for (int u = u_first; u < units && alive; u += u_stride) {
        const Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
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
            const uint32_t d = tmem_base + buf * L::kBufCols;
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              umma_f8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
            umma_commit_pair_both(tfull_bar(buf));
            umma_commit_pair_both(empty_bar(s));
          }
          __syncwarp();
        }
      }
      // every MMA issued above must complete before either CTA frees TMEM or
      // leaves (bounded, and not cut short by the abort flag)
      if (lane == 0) umma_commit_pair_own(drain_bar);
      __syncwarp();
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, p.status);
    }
   } else if constexpr (kUE) {
    // ================================================ MMA issuer, UE8M0 scales
    // The tensor cores apply the scales: each K block's 4 MMAs (kind::mxf8f6f4
    // with block scaling) accumulate into the tile's single TMEM accumulator,
    // which the promotion warps drain once per tile.  Before them, the block's
    // scale words are copied from the stage into TMEM (alternating between
    // two slots), replicated across the four lane quarters; tcgen05 copies and
    // MMAs from this thread execute in order.
    constexpr uint32_t idesc0 = idesc_mxf8_ue8m0(BM, BN);
    const uint32_t acc_t = tmem_base;
    const uint32_t sf_t = tmem_base + static_cast<uint32_t>(L::kBufCols * NBUF);
    int it = 0, tile_i = 0;
    bool alive = true;
    for (int u = u_first; u < units && alive; u += u_stride, ++tile_i) {
      const Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
      // the previous tile's accumulator has been read out
      if (!mbar_wait(tempty_bar(0), (tile_i & 1) ^ 1, s_abort, p.status)) break;
      tc_fence_after();
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(full_bar(s), ph, s_abort, p.status)) { alive = false; break; }
        tc_fence_after();
        if (lane == 0) {
          // the scale words arrived through cp.async (generic proxy); make
          // them visible to the tensor-core copy
          fence_proxy_async_smem();
          const uint32_t sf_s = base + L::kSfOff + static_cast<uint32_t>(s) * kSfStageBytes;
          const uint32_t slot = sf_t + static_cast<uint32_t>(it & 1) * kSfSlotCols;
          tmem_cp_32x128b_x4(slot, smem_desc_rows16(sf_s));
          tmem_cp_32x128b_x4(slot + 4, smem_desc_rows16(sf_s + kSfABytes));
          tmem_cp_32x128b_x4(slot + 8, smem_desc_rows16(sf_s + kSfABytes + 512));
          // byte kb % 4 of each cell holds this K block's scale
          const uint32_t byte = static_cast<uint32_t>(kb & 3);
          const uint32_t idesc = idesc_sf_bytes(idesc0, byte);
          const uint32_t sfa_t = slot | (byte << 30);
          const uint32_t sfb_t = (slot + 4) | (byte << 30);
          const uint32_t sa = base + s * L::kStageBytes;
          const uint64_t adesc = smem_desc_k128_sw128(sa);
          const uint64_t bdesc = smem_desc_k128_sw128(sa + kABytes);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_mxf8_ue8m0(acc_t, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t, sfb_t,
                            (kb > t.k_begin || k > 0) ? 1u : 0u);
          umma_commit(empty_bar(s));
          if (kb + 1 == t.k_end) umma_commit(tfull_bar(0));
        }
        __syncwarp();
      }
    }
   } else {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = idesc_e4m3_f32_major(BM, BN, kAmn, kBmn);
    // advancing one 32-wide K slice: +32 bytes inside a K-major 128-byte row
    // (+2 in the descriptor's 16-byte address field), or +32 rows of 128
    // bytes of an MN-major tile (+256)
    constexpr uint64_t kAStep = kAmn ? 256 : 2, kBStep = kBmn ? 256 : 2;
    int it = 0, acc_it = 0;
    bool alive = true;
    for (int u = u_first; u < units && alive; u += u_stride) {
      Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
      if constexpr (S == kContiguous) {
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
          const uint64_t adesc = kAmn ? smem_desc_mn_sw128(sa, BK * 128)
                                      : smem_desc_k128_sw128(sa);
          const uint64_t bdesc = kBmn ? smem_desc_mn_sw128(sa + kABytes, BK * 128)
                                      : smem_desc_k128_sw128(sa + kABytes);
          const uint32_t d = tmem_base + buf * L::kBufCols;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_f8(d, adesc + kAStep * k, bdesc + kBStep * k, idesc, k > 0 ? 1u : 0u);
          // publish the buffer first: the promotion is on the critical path,
          // the producer has STAGES - 1 blocks of slack
          umma_commit(tfull_bar(buf));
          umma_commit(empty_bar(s));
        }
        __syncwarp();
      }
    }
   }
    if constexpr (!kPair) {
      // every MMA issued above must complete before TMEM is freed (bounded,
      // and not cut short by the abort flag).  (The 2-CTA form drains in its
      // own branch: a kernel's tcgen05 operations all use one CTA group.)
      if (lane == 0) umma_commit(drain_bar);
      __syncwarp();
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, p.status);
    }
  } else if (kStoreWarp && warp == 2) {
    // ============================================================ D stores
    // For each staging use (in the promotion warps' order: the whole tiles,
    // then their column halves), wait until its writers have staged it,
    // store it by TMA, and free the staging tile once the store has read it.
    // Split tiles (reduced through the workspace) stage nothing.
    uint32_t use = 0;
    bool alive = true;
    for (int u = u_first; u < units && alive; u += u_stride) {
      const Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
      if (t.nsplit > 1) continue;
      for (int ph = 0; ph < kStoreUses; ++ph, ++use) {
        if (!mbar_wait(staged_bar, use & 1, s_abort, p.status)) {
          alive = false;
          break;
        }
        if (lane == 0) {
          const int col_base = t.n_blk * BN + ph * 128;
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (col_base + j * static_cast<int>(kStoreBoxCols) < p.n)
              tma_store_3d(&tmap_d, base + L::kOutOff + j * (BM * 128u),
                           col_base + j * kStoreBoxCols,
                           t.m_blk * TM + static_cast<int>(rank) * BM, t.slab);
          bulk_commit_group();
          bulk_wait_group_read_all();  // the staging tile may be written again
          mbar_arrive(free_bar);
        }
        __syncwarp();
      }
    }
    // the stores of D have completed before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }
  } else {
    if constexpr (kRegSplit) setmaxnreg_inc<promo_regs(SCHED)>();
    // ============================================================ promotion
    const int pw = warp - kControlWarps;   // 0..7
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int half = pw >> 2;              // column half of the tile
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const int nb_total = (p.n + 127) / 128;
    int it = 0;
    int tile_i = 0;  // UE8M0: tiles drained so far (the accumulator's phase)
    bool alive = true;
    // every promotion warp arrives once (its lanes' shared-memory writes
    // ordered before lane 0's release by the warp barrier), then all wait for
    // the phase (bounded); the warp agrees on the outcome so that it stays
    // converged for the next sync
    uint32_t epi_phase = 0;
    uint32_t store_use = 0;  // staging uses so far (tiles stored by warp 2)
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      const bool ok = mbar_wait(epi_bar, epi_phase & 1, s_abort, p.status);
      ++epi_phase;
      return __all_sync(0xffffffffu, ok);
    };
    for (int u = u_first; u < units && alive; u += u_stride) {
      Tile t = unit_to_tile(p, S, u, s_prefix, s_mblocks);
      const int row = t.m_blk * TM + static_cast<int>(rank) * BM + row_in_tile;
      bool row_ok;
      if constexpr (S == kContiguous) {
        t.group = block_expert(p, t.m_blk, false);
        if (t.group < 0) continue;
        row_ok = row < p.rows && __ldg(p.m_indices + row) == t.group;
      } else if constexpr (S == kMasked) {
        row_ok = row < masked_rows(p, t.slab);
      } else {
        row_ok = row < p.rows;
      }
      const int col0 = t.n_blk * BN + half * W;  // first column of this thread

      float acc[W];
#pragma unroll
      for (int c = 0; c < W; ++c) acc[c] = 0.0f;

      if constexpr (kUE) {
        // The tensor cores applied the scales and summed the whole K range
        // in TMEM: read this thread's row segment of the accumulator once and
        // hand it back to the MMA warp for the next tile.
        if (!mbar_wait(tfull_bar(0), tile_i & 1, s_abort, p.status)) {
          alive = false;
          break;
        }
        ++tile_i;
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < W; c0 += LW) {
          uint32_t r[LW];
          tmem_ld<LW>(tmem_base + t_lane + half * W + c0, r);
          tmem_wait_ld();
          reg_barrier<LW>(r);
#pragma unroll
          for (int c = 0; c < LW; ++c) acc[c0 + c] = __uint_as_float(r[c]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(0));
      } else {
      // a thread's W columns lie in one beta block when W divides 128 or
      // equals it; a non-power-of-two tile's columns from col0 + cb on take
      // the next block's beta (sfb_ptr1)
      const int nb = min(col0, p.n - 1) / 128;
      const float *sfb_ptr =
          p.sfb + (static_cast<int64_t>(t.group) * nb_total + nb) * kg_total;
      const int cb = kStraddle ? (nb + 1) * 128 - col0 : W;
      const float *sfb_ptr1 =
          kStraddle ? p.sfb + (static_cast<int64_t>(t.group) * nb_total +
                               min(nb + 1, nb_total - 1)) * kg_total
                    : sfb_ptr;

      // This thread's row scale alpha is loaded two K blocks ahead into
      // registers (one coalesced 128-byte load per warp and block); rows past
      // the end read the last row's scale (they are never stored).  The
      // column block's beta, the same for the whole warp, is fetched 32 K
      // blocks at a time, one per lane, a batch ahead, and broadcast with a
      // shuffle.
      const float *a_src = p.sfa + static_cast<int64_t>(t.slab) * kg_total * p.ld_sfa +
                           min(row, p.rows - 1);
      // (a k-grouped tile may have no K blocks: its D is its C)
      float a_cur = !kKG || t.k_begin < t.k_end
                        ? __ldg(a_src + static_cast<int64_t>(t.k_begin) * p.ld_sfa)
                        : 0.0f;
      float a_next = t.k_begin + 1 < t.k_end
                         ? __ldg(a_src + static_cast<int64_t>(t.k_begin + 1) * p.ld_sfa)
                         : 0.0f;
      float b_batch =
          !kKG && t.k_begin + lane < t.k_end ? __ldg(sfb_ptr + t.k_begin + lane) : 0.0f;
      float b_batch_next =
          !kKG && t.k_begin + 32 + lane < t.k_end ? __ldg(sfb_ptr + t.k_begin + 32 + lane)
                                                   : 0.0f;
      float b1_batch =
          kStraddle && t.k_begin + lane < t.k_end ? __ldg(sfb_ptr1 + t.k_begin + lane) : 0.0f;
      float b1_batch_next = kStraddle && t.k_begin + 32 + lane < t.k_end
                                ? __ldg(sfb_ptr1 + t.k_begin + 32 + lane)
                                : 0.0f;
      for (int kb = t.k_begin; kb < t.k_end; ++kb, ++it) {
        float sc = a_cur, sc1 = a_cur;
        if constexpr (!kKG) {
          const int j = (kb - t.k_begin) & 31;
          sc = a_cur * __shfl_sync(0xffffffffu, b_batch, j);
          if constexpr (kStraddle) sc1 = a_cur * __shfl_sync(0xffffffffu, b1_batch, j);
          if (j == 31) {
            b_batch = b_batch_next;
            b_batch_next = kb + 33 + lane < t.k_end ? __ldg(sfb_ptr + kb + 33 + lane) : 0.0f;
            if constexpr (kStraddle) {
              b1_batch = b1_batch_next;
              b1_batch_next = kb + 33 + lane < t.k_end ? __ldg(sfb_ptr1 + kb + 33 + lane) : 0.0f;
            }
          }
        }
        a_cur = a_next;
        if (kb + 2 < t.k_end) a_next = __ldg(a_src + static_cast<int64_t>(kb + 2) * p.ld_sfa);
        const int buf = it % NBUF;
        if (!mbar_wait(tfull_bar(buf), (it / NBUF) & 1, s_abort, p.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        // k-grouped: this block's column scales (landed with the stage that
        // fed the MMA, which completed before tmem_full); this thread's W
        // columns, the same addresses for the whole warp (a broadcast)
        const uint32_t beta_s = kKG ? base + L::kBetaOff +
                                          static_cast<uint32_t>(it % L::kBetaSlots) * (BN * 4u) +
                                          static_cast<uint32_t>(half * W) * 4u
                                    : 0u;
#pragma unroll
        for (int c0 = 0; c0 < W; c0 += LW) {
          uint32_t r[LW];
          tmem_ld<LW>(tmem_base + t_lane + buf * L::kBufCols + half * W + c0, r);
          tmem_wait_ld();
          reg_barrier<LW>(r);
          if constexpr (kKG) {
            // acc += alpha_i * (P_ij * beta_j).  The buffer goes back only
            // after the last scale read: its release lets the MMA warp free
            // the stage whose refill reuses this block's ring slot.
#pragma unroll
            for (int c = 0; c < LW; c += 4) {
              const uint4 bq = ld_shared_v4(beta_s + static_cast<uint32_t>(c0 + c) * 4u);
              float y0 = 0.0f, y1 = 0.0f, y2 = 0.0f, y3 = 0.0f;
              ffma2v(y0, y1, __uint_as_float(r[c]), __uint_as_float(r[c + 1]),
                     __uint_as_float(bq.x), __uint_as_float(bq.y));
              ffma2v(y2, y3, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]),
                     __uint_as_float(bq.z), __uint_as_float(bq.w));
              ffma2(acc[c0 + c], acc[c0 + c + 1], y0, y1, sc);
              ffma2(acc[c0 + c + 2], acc[c0 + c + 3], y2, y3, sc);
            }
            if (c0 + LW == W) {
              // the scale slot is refilled by a bulk copy (async proxy) once
              // the buffer is back: order this thread's generic reads of it
              // before that write (without the fence, repeated runs differed
              // in the last scale reads' columns)
              fence_proxy_async_smem();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty_bar(buf));
            }
          } else {
            if (c0 + LW == W) {
              // all of this buffer has been read: hand it back to the MMA warp
              // (2-CTA form: rank 0's, on its barrier)
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if constexpr (kPair) {
                  mbar_arrive_cluster(mapa_shared(tempty_bar(buf), 0));
                } else {
                  mbar_arrive(tempty_bar(buf));
                }
              }
            }
            const float s_chunk = !kStraddle || c0 < cb ? sc : sc1;
#pragma unroll
            for (int c = 0; c < LW; c += 2)
              ffma2(acc[c0 + c], acc[c0 + c + 1], __uint_as_float(r[c]), __uint_as_float(r[c + 1]),
                    s_chunk);
          }
        }
      }
      }  // (not UE8M0)
      if (!alive) break;

      // ---------------------------------------------------------- epilogue
      // (split K serves dense shapes only; the grouped instances leave it
      // out, which also keeps their register allocation lean)
      if (kDenseLike && t.nsplit > 1) {
        if (*s_abort) break;
        // Split K: every CTA of the tile writes its FP32 partial (valid rows
        // only, as float4 slots [column / 4][row] so that a warp's 32 rows
        // write 512 contiguous bytes), counts itself in on the tile's
        // arrival counter and waits for all splits (the launch is
        // cooperative, so they are all resident); then each split reduces its
        // own 1/S share of the tile's slots, summing splits 0, 1, ... in
        // order (deterministic), and stores that share as BF16.
        const int tile = t.tile - p.full_tiles;  // index among the split tiles
        constexpr int kTileSlots = BM * BN / 4;
        float4 *part = reinterpret_cast<float4 *>(p.ws) +
                       static_cast<int64_t>(tile) * p.splits * kTileSlots;
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < W; c += 4)
            __stcg(part + static_cast<int64_t>(t.split) * kTileSlots +
                       ((half * W + c) / 4) * BM + row_in_tile,
                   make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
        }
        __threadfence();
        if (!epi_sync()) break;
        const int ptid = threadIdx.x - kControlWarps * 32;
        if (ptid == 0) {
          atomicAdd(p.ws_ticket + tile, 1u);
          if (!wait_counter(p.ws_ticket + tile, static_cast<uint32_t>(p.splits), p.status))
            *s_abort = 1;
        }
        if (!epi_sync()) break;
        if (*s_abort) break;
        __threadfence();
        const int row0 = t.m_blk * BM;
        const int valid = min(BM, p.rows - row0);
        const int slots = valid * (BN / 4);
        const int share = (slots + p.splits - 1) / p.splits;
        const int f_end = min(slots, (t.split + 1) * share);
        // Q slots per thread per pass so that their loads overlap; each
        // slot is summed over splits 0, 1, ... in order (deterministic)
        constexpr int Q = 4;
        for (int f0 = t.split * share + ptid; f0 < f_end; f0 += Q * kPromoThreads) {
          const float4 *src[Q];
          bool ok[Q];
          float4 sum[Q];
#pragma unroll
          for (int q = 0; q < Q; ++q) {
            const int f = f0 + q * kPromoThreads;
            ok[q] = f < f_end;
            const int c4 = ok[q] ? f / valid : 0;
            src[q] = part + c4 * BM + (ok[q] ? f - c4 * valid : 0);
            sum[q] = ok[q] ? __ldcg(src[q]) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll 2
          for (int s = 1; s < p.splits; ++s) {
            float4 v[Q];
#pragma unroll
            for (int q = 0; q < Q; ++q)
              v[q] = ok[q] ? __ldcg(src[q] + static_cast<int64_t>(s) * kTileSlots)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < Q; ++q) {
              sum[q].x += v[q].x;
              sum[q].y += v[q].y;
              sum[q].z += v[q].z;
              sum[q].w += v[q].w;
            }
          }
#pragma unroll
          for (int q = 0; q < Q; ++q) {
            const int f = f0 + q * kPromoThreads;
            const int c4 = f / valid, r = f - c4 * valid;
            const int col = t.n_blk * BN + 4 * c4;
            if (ok[q] && col < p.n) {
              if constexpr (S == kDenseAcc) {
                const float4 cv = __ldg(reinterpret_cast<const float4 *>(
                    p.c + static_cast<int64_t>(row0 + r) * p.n + col));
                sum[q].x += cv.x;
                sum[q].y += cv.y;
                sum[q].z += cv.z;
                sum[q].w += cv.w;
              }
              const __nv_bfloat162 lo = __floats2bfloat162_rn(sum[q].x, sum[q].y);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(sum[q].z, sum[q].w);
              uint2 v;
              v.x = *reinterpret_cast<const uint32_t *>(&lo);
              v.y = *reinterpret_cast<const uint32_t *>(&hi);
              *reinterpret_cast<uint2 *>(p.d + static_cast<int64_t>(row0 + r) * p.n + col) = v;
            }
          }
        }
        continue;  // this split's share of D is written
      }
      if constexpr (kKG) {
        // D[g] = C[g] + A_g B_g^T in FP32: each thread stores its row
        // segment, 16 bytes at a time, adding the matching 16 bytes of C
        if (row_ok) {
          const int64_t off = (static_cast<int64_t>(t.group) * p.rows + row) * p.n;
          float *drow = p.d_f32 + off;
#pragma unroll
          for (int c = 0; c < W; c += 4) {
            if (col0 + c < p.n) {
              float4 v = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
              if (p.c != nullptr) {
                const float4 cv = __ldg(reinterpret_cast<const float4 *>(p.c + off + col0 + c));
                v.x += cv.x;
                v.y += cv.y;
                v.z += cv.z;
                v.w += cv.w;
              }
              *reinterpret_cast<float4 *>(drow + col0 + c) = v;
            }
          }
        }
        continue;
      }
      if constexpr (S == kDenseCluster) {
        // Leave this split's FP32 partial in this CTA's shared memory (the
        // stage ring, drained: every block's MMAs have completed) for the
        // cluster reduction after the role loops.  Layout [128 rows][BN/4]
        // 16-byte chunks, chunk c of row r at c ^ (r mod kSwF): the
        // row-per-lane writes and the row-major reads are both conflict-free.
        constexpr int kChunksF = BN / 4;
        constexpr int kSwF = kChunksF < 8 ? kChunksF : 8;
        float4 *s_part = reinterpret_cast<float4 *>(smem);
#pragma unroll
        for (int c = 0; c < W; c += 4) {
          const int chunk = (half * W + c) / 4;
          s_part[row_in_tile * kChunksF + (chunk ^ (row_in_tile % kSwF))] =
              make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        }
        continue;  // one unit per CTA in this schedule
      }
      if constexpr (kQ) {
        // D quantized 1 x 128 along N: this thread's 128 columns are one
        // group of its row.  As the 1x128 quantizer would do on the BF16
        // result: round to BF16, amax, s = amax / 448 (or its power of two
        // above), codes E4M3_RNE(x / s); the codes go out 16 bytes at a time
        // and the scale to the MN-major [N/128][ld] layout (consecutive rows
        // of a warp: one 128-byte store).
        if (row_ok && col0 < p.n) {
          float amax = 0.0f;
#pragma unroll
          for (int c = 0; c < W; ++c) {
            acc[c] = __bfloat162float(__float2bfloat16_rn(acc[c]));
            amax = fmaxf(amax, fabsf(acc[c]));
          }
          const float sc = group_scale(amax, p.q_flags);
          const bool fast = sc >= kFastDivMin;
          const float y = fast ? __frcp_rn(sc) : 0.0f;
          uint8_t *qrow = p.dq + static_cast<int64_t>(row) * p.n + col0;
#pragma unroll
          for (int c = 0; c < W; c += 16) {
            uint4 w;
            w.x = encode4(acc + c, sc, y, fast);
            w.y = encode4(acc + c + 4, sc, y, fast);
            w.z = encode4(acc + c + 8, sc, y, fast);
            w.w = encode4(acc + c + 12, sc, y, fast);
            *reinterpret_cast<uint4 *>(qrow + c) = w;
          }
          p.sfd[static_cast<int64_t>(col0 / 128) * p.ld_sfd + row] = sc;
        }
      } else if constexpr (!kStaged) {
        // each thread stores its row segment (valid rows), 16 bytes at a time
        if (row_ok) {
          uint16_t *drow = p.d + (static_cast<int64_t>(t.slab) * p.rows + row) * p.n;
#pragma unroll
          for (int c = 0; c < W; c += 8) {
            if (col0 + c < p.n) {
              uint4 v;
              uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 h =
                    __floats2bfloat162_rn(acc[c + 2 * j], acc[c + 2 * j + 1]);
                w[j] = *reinterpret_cast<const uint32_t *>(&h);
              }
              *reinterpret_cast<uint4 *>(drow + col0 + c) = v;
            }
          }
        }
      } else if constexpr (kStaged == 2) {
        // D = C + A B^T: the FP32 tile goes through shared memory in 64-column
        // phases ([128 rows][kOutCols] FP32, 16-byte chunk c of row r at
        // c ^ (r mod kSw)); on the way out each lane adds the matching 16
        // bytes of C (consecutive lanes read consecutive columns of a row),
        // rounds the sum to BF16 and stores 8 bytes.
        constexpr int kChunks = L::kOutCols / 4;        // 16-byte chunks per staged row
        constexpr int kSw = kChunks < 8 ? kChunks : 8;
        constexpr int kPhases = BN / L::kOutCols;
        constexpr int kRowBytes = L::kOutCols * 4;
        const uint32_t s_out = base + L::kOutOff;
        uint8_t *s_rowok = smem + L::kRowOkOff;
        const int ptid = threadIdx.x - kControlWarps * 32;
        const int64_t row0 = static_cast<int64_t>(t.m_blk) * BM;
        if (half == 0) s_rowok[row_in_tile] = row_ok ? 1 : 0;
#pragma unroll
        for (int ph = 0; ph < kPhases; ++ph) {
#pragma unroll
          for (int c = 0; c < W; c += 4) {
            const int tcol = half * W + c;  // tile column of acc[c]
            if (tcol / L::kOutCols == ph) {
              const int chunk = (tcol % L::kOutCols) / 4;
              st_shared_v4(s_out + row_in_tile * kRowBytes + ((chunk ^ (row_in_tile % kSw)) * 16),
                           __float_as_uint(acc[c]), __float_as_uint(acc[c + 1]),
                           __float_as_uint(acc[c + 2]), __float_as_uint(acc[c + 3]));
            }
          }
          if (!epi_sync()) {
            alive = false;
            break;
          }
          const int col_base = t.n_blk * BN + ph * L::kOutCols;
          // unrolled so that the read-only loads of C of several iterations
          // are in flight together
#pragma unroll 4
          for (int f = ptid; f < BM * kChunks; f += kPromoThreads) {
            const int r = f / kChunks, ch = f - r * kChunks;
            const int col = col_base + ch * 4;
            if (s_rowok[r] && col < p.n) {
              const uint4 a = ld_shared_v4(s_out + r * kRowBytes + ((ch ^ (r % kSw)) * 16));
              const int64_t off = (row0 + r) * p.n + col;
              const float4 cv = __ldg(reinterpret_cast<const float4 *>(p.c + off));
              const __nv_bfloat162 lo =
                  __floats2bfloat162_rn(__uint_as_float(a.x) + cv.x, __uint_as_float(a.y) + cv.y);
              const __nv_bfloat162 hi =
                  __floats2bfloat162_rn(__uint_as_float(a.z) + cv.z, __uint_as_float(a.w) + cv.w);
              uint2 v;
              v.x = *reinterpret_cast<const uint32_t *>(&lo);
              v.y = *reinterpret_cast<const uint32_t *>(&hi);
              *reinterpret_cast<uint2 *>(p.d + off) = v;
            }
          }
          if (!epi_sync()) {
            alive = false;
            break;
          }
        }
      } else {
        // The tile leaves through shared memory.  Staging layout: [128 rows]
        // x kOutCols BF16; a 128-column half is two boxes of [128 rows][64
        // columns], 128 bytes a row, 16-byte chunk c of row r at c ^ (r mod 8)
        // -- the 128-byte swizzle of the TMA store's tensor map, and free of
        // bank conflicts both for the row-per-lane writes and for row-major
        // reads.  A 256-wide tile goes out in two column halves, each written
        // by the warps that own it.  Dense tiles leave by TMA stores issued
        // by one thread, and so do UE8M0 masked tiles whose rows are all
        // valid; other masked tiles (rows past an expert's count stay
        // untouched) leave by warp stores of whole row segments, valid rows
        // only.
        constexpr int kChunks = L::kOutCols / 8;        // 16-byte chunks per staged row
        constexpr int kSw = kChunks < 8 ? kChunks : 8;  // swizzle span, in chunks
        // phases of kOutCols columns: one (a 128-wide or narrower tile), one
        // per column half (256 wide, 128-column staging), or two per half
        // (256 wide, 64-column staging: the UE8M0 forms)
        constexpr int kPhases = BN > static_cast<int>(L::kOutCols) ? BN / L::kOutCols : 1;
        constexpr int kPhasesPerHalf = kPhases > 1 ? kPhases / 2 : 1;
        constexpr int kRowBytes = kChunks < 8 ? L::kOutCols * 2 : 128;
        auto staged_off = [&](int r, int c) -> uint32_t {
          return static_cast<uint32_t>((c / kSw) * (BM * kRowBytes) + r * kRowBytes +
                                       ((c % kSw) ^ (r % kSw)) * 16);
        };
        const uint32_t s_out = base + L::kOutOff;
        uint8_t *s_rowok = smem + L::kRowOkOff;
        const int ptid = threadIdx.x - kControlWarps * 32;
        const int64_t slab_row0 = static_cast<int64_t>(t.slab) * p.rows + t.m_blk * TM +
                                  static_cast<int>(rank) * BM;
        if constexpr (kStoreWarp) {
          // This warp's staging use: wait until the previous use's TMA
          // store has read the staging tile, write the columns, make them
          // visible to the async proxy and hand the use to warp 2.
#pragma unroll
          for (int ph = 0; ph < kStoreUses; ++ph) {
            if (kStoreUses == 1 || half == ph) {
              const uint32_t use = store_use + static_cast<uint32_t>(ph);
              bool ok = use == 0 || mbar_wait(free_bar, (use - 1) & 1, s_abort, p.status);
              if (!__all_sync(0xffffffffu, ok)) {
                alive = false;
                break;
              }
              const int scol0 = kStoreUses == 1 ? half * W : 0;  // staged column of acc[0]
#pragma unroll
              for (int c = 0; c < W; c += 8) {
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const __nv_bfloat162 h =
                      __floats2bfloat162_rn(acc[c + 2 * j], acc[c + 2 * j + 1]);
                  w[j] = *reinterpret_cast<const uint32_t *>(&h);
                }
                st_shared_v4(s_out + staged_off(row_in_tile, (scol0 + c) / 8), w[0], w[1], w[2],
                             w[3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(staged_bar);
            }
          }
          store_use += kStoreUses;
          if (!alive) break;
          continue;
        }
        const bool tma_tile =
            kTmaStore && (S == kDense || (t.m_blk + 1) * BM <= masked_rows(p, t.slab));
        if (!tma_tile && half == 0) s_rowok[row_in_tile] = row_ok ? 1 : 0;
#pragma unroll
        for (int ph = 0; ph < kPhases; ++ph) {
          // the phase's columns belong to half ph / kPhasesPerHalf, slice
          // ph % kPhasesPerHalf of each of its threads' W columns
          if (kPhases == 1 || half == ph / kPhasesPerHalf) {
            const int sub = kPhases == 1 ? 0 : ph % kPhasesPerHalf;
#pragma unroll
            for (int c = 0; c < W; c += 8) {
              if (kPhases > 1 && c / static_cast<int>(L::kOutCols) != sub) continue;
              uint32_t w[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(acc[c + 2 * j], acc[c + 2 * j + 1]);
                w[j] = *reinterpret_cast<const uint32_t *>(&h);
              }
              // staged column of acc[c]: the thread's own (one phase) or its
              // place in the phase's kOutCols
              const int scol = kPhases == 1 ? half * W + c : c % static_cast<int>(L::kOutCols);
              st_shared_v4(s_out + staged_off(row_in_tile, scol / 8), w[0], w[1], w[2], w[3]);
            }
            // the TMA store reads the tile through the async proxy
            if constexpr (kTmaStore) fence_proxy_async_smem();
          }
          if (!epi_sync()) {
            alive = false;
            break;
          }
          const int col_base = t.n_blk * BN + ph * static_cast<int>(L::kOutCols);
          if (tma_tile) {
            if (ptid == 0) {
#pragma unroll
              for (int j = 0; j < (kChunks + 7) / 8; ++j)
                if (col_base + j * static_cast<int>(kStoreBoxCols) < p.n)
                  tma_store_3d(&tmap_d, s_out + j * (BM * 128u), col_base + j * kStoreBoxCols,
                               t.m_blk * TM + static_cast<int>(rank) * BM, t.slab);
              bulk_commit_group();
              bulk_wait_group_read_all();  // the staging tile may be written again
            }
          } else {
#pragma unroll 1
            for (int f = ptid; f < BM * kChunks; f += kPromoThreads) {
              const int r = f / kChunks, ch = f - r * kChunks;
              const int col = col_base + ch * 8;
              if (s_rowok[r] && col < p.n) {
                const uint4 v = ld_shared_v4(s_out + staged_off(r, ch));
                *reinterpret_cast<uint4 *>(p.d + (slab_row0 + r) * p.n + col) = v;
              }
            }
          }
          if (!epi_sync()) {
            alive = false;
            break;
          }
        }
      }
      if (!alive) break;
    }
    // the TMA stores of D have completed before the CTA exits
    if constexpr (kTmaStore) {
      if (threadIdx.x == kControlWarps * 32) bulk_wait_group_all();
    }
  }

  // ------------------------------------------------ cluster split reduction
  // The splits of a tile are the CTAs of one cluster (rank = split).  Every
  // thread of every CTA passes both cluster barriers, whatever happened in
  // its role loop, so none can strand the others.
  if constexpr (S == kDenseCluster) {
    __syncwarp();
    cluster_sync();  // all partials written
    if (warp >= kControlWarps && !*s_abort) {
      const Tile t = unit_to_tile(p, S, static_cast<int>(blockIdx.x), s_prefix, s_mblocks);
      constexpr int kChunksF = BN / 4;
      constexpr int kSwF = kChunksF < 8 ? kChunksF : 8;
      const int split = static_cast<int>(cluster_ctarank());
      const int row0 = t.m_blk * BM;
      const int valid = min(BM, p.rows - row0);
      const int total = valid * kChunksF;  // row-major chunks of the valid rows
      const int share = (total + p.splits - 1) / p.splits;
      const int f_end = min(total, (split + 1) * share);
      const int ptid = threadIdx.x - kControlWarps * 32;
      for (int f = split * share + ptid; f < f_end; f += kPromoThreads) {
        const int r = f / kChunksF, c = f - r * kChunksF;
        const uint32_t off = base + 16u * (r * kChunksF + (c ^ (r % kSwF)));
        // every split's chunk in flight at once, then summed in split order
        // (deterministic); a cluster has at most kMaxClusterSplits CTAs
        float4 v[kMaxClusterSplits];
#pragma unroll
        for (int q = 0; q < kMaxClusterSplits; ++q)
          if (q < p.splits) v[q] = ld_shared_cluster_v4(mapa_shared(off, static_cast<uint32_t>(q)));
        float4 sum = v[0];
#pragma unroll
        for (int q = 1; q < kMaxClusterSplits; ++q) {
          if (q < p.splits) {
            sum.x += v[q].x;
            sum.y += v[q].y;
            sum.z += v[q].z;
            sum.w += v[q].w;
          }
        }
        const int col = t.n_blk * BN + 4 * c;
        if (col < p.n) {
          const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
          const __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
          uint2 v;
          v.x = *reinterpret_cast<const uint32_t *>(&lo);
          v.y = *reinterpret_cast<const uint32_t *>(&hi);
          *reinterpret_cast<uint2 *>(p.d + static_cast<int64_t>(row0 + r) * p.n + col) = v;
        }
      }
    }
    cluster_sync();  // no CTA leaves while its partial is being read
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // 2-CTA form: neither CTA leaves or frees TMEM while rank 0's MMAs may
  // still read its shared memory or write its TMEM (rank 0 drained them)
  if constexpr (kPair) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_dealloc_pair(tmem_base, L::kTmemCols);
    } else {
      tmem_dealloc(tmem_base, L::kTmemCols);
    }
  }
}

// ------------------------------------------------------------------ host side
struct Candidate {
  int bn, stages, nbuf;
};
// N tiles and their pipeline depths: 4-6 stages keep ~200 KB of operands in
// flight; NBUF fills the 512 TMEM columns (at most 8 buffers).
constexpr Candidate kCandidates[] = {
    {256, 4, 2}, {128, 6, 4}, {64, 8, 8}, {32, 8, 8}, {16, 8, 8}};

// Tile forms of the cluster split (decode-sized dense NT shapes): the
// power-of-two forms above and non-power-of-two widths, which let more of
// the SMs stream B when the power-of-two tiling leaves clusters that do not
// fit one wave.  Stages: as many as fit the shared memory (more blocks in
// flight per SM).
constexpr Candidate kClusterForms[] = {{256, 4, 2}, {224, 5, 2}, {192, 5, 2}, {160, 6, 2},
                                       {128, 6, 4}, {96, 7, 4},  {64, 8, 8}};

// Whether dense NT launches of two or more M blocks take the 2-CTA form
// unless DG_PAIR says otherwise.
constexpr bool kPairByDefault = false;

// The UE8M0 schedules' one tile form: 256 wide, one accumulator (the tile
// sums all of K in TMEM), four stages (beside the per-stage scale-factor
// areas and a 64-column output staging tile).
constexpr Candidate kUECandidate = {256, 4, 1};

template <int BN, int STAGES, int NBUF, int STAGED, bool KG = false, bool UE = false,
          bool PAIR = false>
constexpr int smem_bytes_for(int extra) {
  return 1024 + Layout<BN, STAGES, NBUF, STAGED, KG, UE, PAIR>::kTableOff + extra;
}

bool print_configs() {
  const char *e = getenv("DG_PRINT_CONFIGS");
  return e && *e && *e != '0';
}

// Sets the instance's dynamic shared memory limit (once per device, grows
// only); false on a CUDA error.
template <int BN, int STAGES, int NBUF, int SCHED, int LAYOUT>
bool configure_smem(int smem) {
  static int configured_smem[64] = {0};  // per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (smem > configured_smem[dev]) {
    if (cudaFuncSetAttribute(fp8_gemm_kernel<BN, STAGES, NBUF, SCHED, LAYOUT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return false;
    configured_smem[dev] = smem;
  }
  return true;
}

template <int BN, int STAGES, int NBUF, int SCHED>
constexpr int instance_smem(int extra) {
  return smem_bytes_for<BN, STAGES, NBUF, instance_staging(SCHED), SCHED == kKGrouped,
                        is_ue8m0(SCHED), SCHED == kDensePair>(extra);
}

// How many thread-block clusters of `cluster` CTAs of this instance can be
// resident at once (the occupancy calculator, cached per device; 0 when the
// size is unsupported or the query fails).
template <int BN, int STAGES, int NBUF, int SCHED, int LAYOUT>
int clusters_fit(int cluster) {
  static int fit[64][kMaxClusterSplits + 1] = {};  // max active clusters + 1; 0 = not asked
  int dev = 0;
  if (cluster < 2 || cluster > kMaxClusterSplits || cudaGetDevice(&dev) != cudaSuccess ||
      dev < 0 || dev >= 64)
    return 0;
  if (fit[dev][cluster] == 0) {
    const int smem = instance_smem<BN, STAGES, NBUF, SCHED>(0);
    int n = 0;
    if (configure_smem<BN, STAGES, NBUF, SCHED, LAYOUT>(smem)) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(cluster);
      q.blockDim = dim3(kThreads);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = cluster;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      const cudaError_t e =
          cudaOccupancyMaxActiveClusters(&n, fp8_gemm_kernel<BN, STAGES, NBUF, SCHED, LAYOUT>, &q);
      if (e != cudaSuccess) {
        cudaGetLastError();  // clear: the caller takes another form
        n = 0;
      }
      if (print_configs())
        fprintf(stderr, "[dg] BN=%d clusters of %d: at most %d resident (%s)\n", BN, cluster, n,
                cudaGetErrorString(e));
    } else {
      cudaGetLastError();
    }
    fit[dev][cluster] = n + 1;
  }
  return fit[dev][cluster] - 1;
}

template <int BN, int STAGES, int NBUF, int SCHED, int LAYOUT = kLayoutNT>
int launch_instance(const CUtensorMap &ta, const CUtensorMap &tb,
                    const CUtensorMap &td, const GemmParams &p,
                    int grid, int extra_smem, cudaStream_t stream, bool coop) {
  const int smem = instance_smem<BN, STAGES, NBUF, SCHED>(extra_smem);
  auto kern = fp8_gemm_kernel<BN, STAGES, NBUF, SCHED, LAYOUT>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DG_ERR_CUDA;
  if constexpr (uses_reg_split(BN, base_sched(SCHED))) {
    // the warpgroup register split needs the full launch allocation: never
    // launch an instance compiled to fewer registers (its promotion warps
    // would wait for registers that never come)
    static int regs_checked = 0;  // 1 ok, -1 too few
    if (regs_checked == 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return DG_ERR_CUDA;
      regs_checked = fa.numRegs >= kLaunchRegs ? 1 : -1;
    }
    if (regs_checked < 0) return DG_ERR_CUDA;
  }
  if (!configure_smem<BN, STAGES, NBUF, SCHED, LAYOUT>(smem)) return DG_ERR_CUDA;
  // clusters: the `splits` CTAs of a tile, or the CTA pair
  const int cluster = SCHED == kDenseCluster ? p.splits : SCHED == kDensePair ? 2 : 1;
  if constexpr (SCHED == kDenseCluster) {
    // every cluster must be resident at once (one wave)
    if (grid / cluster > clusters_fit<BN, STAGES, NBUF, SCHED, LAYOUT>(cluster)) return kClusterNoFit;
  }
  int launch_grid = grid;
  if constexpr (SCHED == kDensePair) {
    // a persistent grid of pairs: never more pairs than fit at once (clusters
    // of two need two free SMs of one GPC; a pair that is not resident would
    // only start once another has finished all its tiles)
    static int pairs_fit[64] = {};  // max active clusters + 1; 0 = not asked yet
    if (pairs_fit[dev] == 0) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(grid);
      q.blockDim = dim3(kThreads);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 2;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      if (print_configs()) fprintf(stderr, "[dg] 2-CTA form: at most %d pairs resident\n", n);
      pairs_fit[dev] = n + 1;
    }
    const int fit = pairs_fit[dev] - 1;
    if (fit < 1) return DG_ERR_CUDA;
    launch_grid = 2 * std::min(grid / 2, fit);
  }
  if (coop) {
    // the splits of a tile wait for each other: all CTAs must be resident
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, td, p) != cudaSuccess) return DG_ERR_CUDA;
  } else {
    // programmatic dependent launch: the kernel's set-up overlaps the tail of
    // the previous kernel (it waits for that grid before touching memory)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(launch_grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0] = pdl_attribute();
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster > 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = cluster;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
    }
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, td, p) != cudaSuccess) return DG_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

// Clusters of `cluster` CTAs of the cluster-split instance of width `bn`
// that fit at once (0 for a width without an instance).
int cluster_split_fit(int bn, int cluster) {
  switch (bn) {
    case 256: return clusters_fit<256, 4, 2, kDenseCluster, kLayoutNT>(cluster);
    case 224: return clusters_fit<224, 5, 2, kDenseCluster, kLayoutNT>(cluster);
    case 192: return clusters_fit<192, 5, 2, kDenseCluster, kLayoutNT>(cluster);
    case 160: return clusters_fit<160, 6, 2, kDenseCluster, kLayoutNT>(cluster);
    case 128: return clusters_fit<128, 6, 4, kDenseCluster, kLayoutNT>(cluster);
    case 96: return clusters_fit<96, 7, 4, kDenseCluster, kLayoutNT>(cluster);
    case 64: return clusters_fit<64, 8, 8, kDenseCluster, kLayoutNT>(cluster);
    default: return 0;
  }
}

// Dynamic shared memory of a single-CTA tile form for a schedule (extra =
// its prefix tables).
template <int BN, int STAGES, int NBUF>
int single_smem(int sched, int extra) {
  switch (staged_epilogue(sched)) {
    case 1: return smem_bytes_for<BN, STAGES, NBUF, 1>(extra);
    case 2: return smem_bytes_for<BN, STAGES, NBUF, 2>(extra);
    default:
      return sched == kKGrouped ? smem_bytes_for<BN, STAGES, NBUF, 0, true>(extra)
                                : smem_bytes_for<BN, STAGES, NBUF, 0>(extra);
  }
}

int config_smem(int bn, int extra, int sched) {
  if (is_ue8m0(sched))
    // (both UE8M0 schedules stage the BF16 tile 64 columns at a time: kind 3)
    return smem_bytes_for<kUECandidate.bn, kUECandidate.stages, kUECandidate.nbuf,
                          instance_staging(kDenseUE8M0), false, true>(extra);
  switch (bn) {
    case 256: return single_smem<256, 4, 2>(sched, extra);
    case 128: return single_smem<128, 6, 4>(sched, extra);
    case 64: return single_smem<64, 8, 8>(sched, extra);
    case 32: return single_smem<32, 8, 8>(sched, extra);
    case 16: return single_smem<16, 8, 8>(sched, extra);
    default: break;
  }
  if (sched != kDenseCluster) return 1 << 30;
  switch (bn) {  // the cluster split's non-power-of-two widths
    case 224: return single_smem<224, 5, 2>(sched, extra);
    case 192: return single_smem<192, 5, 2>(sched, extra);
    case 160: return single_smem<160, 6, 2>(sched, extra);
    case 96: return single_smem<96, 7, 4>(sched, extra);
    default: return 1 << 30;
  }
}

// The opt-in shared memory limit per block of the current device.
int max_smem_per_block() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 232448;  // B200
  return v;
}

// The transposed layouts: tiles 256 or 128 wide (a whole number of
// 128-value MN-major columns of B).
template <int SCHED, int LAYOUT>
int dispatch_layout(int bn, const CUtensorMap &ta, const CUtensorMap &tb,
                    const CUtensorMap &td, const GemmParams &p,
                    int grid, int extra, cudaStream_t st) {
  const bool coop = p.splits > 1 && SCHED != kDenseCluster;
  switch (bn) {
    case 256: return launch_instance<256, 4, 2, SCHED, LAYOUT>(ta, tb, td, p, grid, extra, st, coop);
    case 128: return launch_instance<128, 6, 4, SCHED, LAYOUT>(ta, tb, td, p, grid, extra, st, coop);
    default: return DG_ERR_INVALID_ARG;
  }
}

template <int SCHED>
int dispatch_any_layout(int layout, int bn, const CUtensorMap &ta, const CUtensorMap &tb,
                    const CUtensorMap &td,
                        const GemmParams &p, int grid, int extra, cudaStream_t st) {
  switch (layout) {
    case kLayoutNN: return dispatch_layout<SCHED, kLayoutNN>(bn, ta, tb, td, p, grid, extra, st);
    case kLayoutTN: return dispatch_layout<SCHED, kLayoutTN>(bn, ta, tb, td, p, grid, extra, st);
    case kLayoutTT: return dispatch_layout<SCHED, kLayoutTT>(bn, ta, tb, td, p, grid, extra, st);
    default: return DG_ERR_INVALID_ARG;
  }
}

template <int SCHED>
int dispatch(int bn, const CUtensorMap &ta, const CUtensorMap &tb,
                    const CUtensorMap &td, const GemmParams &p,
             int grid, int extra, cudaStream_t st) {
  if constexpr (SCHED == kDenseCluster) {
    // the non-power-of-two widths (cluster split, NT only)
    switch (bn) {
      case 224: return launch_instance<224, 5, 2, SCHED>(ta, tb, td, p, grid, extra, st, false);
      case 192: return launch_instance<192, 5, 2, SCHED>(ta, tb, td, p, grid, extra, st, false);
      case 160: return launch_instance<160, 6, 2, SCHED>(ta, tb, td, p, grid, extra, st, false);
      case 96: return launch_instance<96, 7, 4, SCHED>(ta, tb, td, p, grid, extra, st, false);
      default: break;
    }
  }
  // splits that wait for each other through global memory need all CTAs
  // resident; a cluster's splits are co-scheduled by construction
  const bool coop = p.splits > 1 && SCHED != kDenseCluster;
  if constexpr (is_ue8m0(SCHED)) {
    return launch_instance<kUECandidate.bn, kUECandidate.stages, kUECandidate.nbuf, SCHED>(
        ta, tb, td, p, grid, extra, st, false);
  } else if constexpr (SCHED == kDenseQuant) {
    return launch_instance<256, 4, 2, SCHED>(ta, tb, td, p, grid, extra, st, false);
  } else if constexpr (SCHED == kDensePair) {
    // 32 KB stages (A 16 KB + half of B 16 KB): six fit beside the staging
    return launch_instance<256, 6, 2, SCHED>(ta, tb, td, p, grid, extra, st, false);
  } else {
    switch (bn) {
      case 256: return launch_instance<256, 4, 2, SCHED>(ta, tb, td, p, grid, extra, st, coop);
      case 128: return launch_instance<128, 6, 4, SCHED>(ta, tb, td, p, grid, extra, st, coop);
      case 64: return launch_instance<64, 8, 8, SCHED>(ta, tb, td, p, grid, extra, st, coop);
      case 32: return launch_instance<32, 8, 8, SCHED>(ta, tb, td, p, grid, extra, st, coop);
      case 16: return launch_instance<16, 8, 8, SCHED>(ta, tb, td, p, grid, extra, st, coop);
      default: return DG_ERR_INVALID_ARG;
    }
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


// 3-D tensor map over an E4M3 tensor stored [dim2][K][rows] (K outermost
// within a slab: an MN-major operand) with a box of [1][128][128] (128 K rows
// of 128 values) and the 128-byte swizzle.  rows % 16 == 0 (the row stride of
// a TMA tensor is a multiple of 16 bytes).
int make_tmap_mn(CUtensorMap *m, const void *ptr, int64_t rows, int64_t k, int64_t slabs) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return DG_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(k),
                              static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(rows),
                                 static_cast<cuuint64_t>(rows * k)};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(BK), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 3-D tensor map over the BF16 output D [slabs][rows][n] for the epilogue's
// TMA stores: a box of [1][128 rows][64 columns] (128 bytes, the staging
// tile's 128-byte swizzle).  n % 8 == 0 and D 16-byte aligned (checked by
// the entry points), so the row stride is a multiple of 16 bytes.
int make_tmap_d(CUtensorMap *m, void *d, int64_t rows, int64_t n, int64_t slabs) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return DG_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(n * 2),
                                 static_cast<cuuint64_t>(n * rows * 2)};
  const cuuint32_t box[3] = {kStoreBoxCols, BM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, d, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// Cycles one CTA spends per 128-K block of a unit, measured on B200.  The
// tensor cores take ~540 cycles per block for any N up to 256 (one
// 128 x N x 32 MMA per ~135 cycles), so narrow tiles waste them; the
// MMA -> promotion -> MMA round trip through the TMEM buffers sets the rest.
double kb_cycles(int bn) {
  switch (bn) {
    case 256: return 1240.0;
    case 224: return 1160.0;  // (non-power-of-two widths: interpolated)
    case 192: return 1070.0;
    case 160: return 990.0;
    case 128: return 900.0;
    case 96: return 830.0;
    case 64: return 770.0;
    default: return 750.0;
  }
}

// Estimated time (SM cycles) of a config: waves x per-unit time (K blocks x
// kb_cycles + pipeline fill and epilogue + split-K reduction), floored by
// streaming the distinct operand bytes once through HBM (~23 B/cycle/SM).
double estimate(int64_t m_blocks, int64_t n, int64_t k, int bn, int splits, int sms) {
  const int64_t n_blocks = (n + bn - 1) / bn;
  const int64_t units = m_blocks * n_blocks * splits;
  const int64_t waves = (units + sms - 1) / sms;
  const int64_t kb = (k / BK + splits - 1) / splits;
  double per_unit = kb * kb_cycles(bn) + 2500.0;
  if (splits > 1) per_unit += 1500.0 + 300.0 * splits;
  const double t = waves * per_unit;
  const double bytes = static_cast<double>(n) * k + m_blocks * 128.0 * k;
  return std::max(t, bytes / (23.0 * sms));
}

// The cluster split of a decode-sized shape streams B through every CTA's
// stage ring: a CTA completes about one K block per kLoadLatency / STAGES
// cycles (each block's copy takes a loaded-memory round trip; STAGES are in
// flight; measured ~2.9 us per round trip with the 4-stage 256-wide form on
// B200), never faster than its tensor work, and the launch never moves its
// bytes faster than HBM (~3,400 bytes per SM cycle).
constexpr double kLoadLatency = 5600.0;
constexpr double kHbmBytesPerCycle = 3400.0;

double estimate_cluster(int64_t m_blocks, int64_t n, int64_t k, const Candidate &f, int s) {
  const int64_t kb = (k / BK + s - 1) / s;
  const double per_kb = std::max(kb_cycles(f.bn), kLoadLatency / f.stages);
  const double t = kb * per_kb + 2500.0 + 1500.0 + 300.0 * s;
  const double bytes = static_cast<double>(n) * k + m_blocks * 128.0 * k;
  return std::max(t, bytes / kHbmBytesPerCycle);
}

// The cluster split's form for a decode-sized dense NT shape: the width and
// split of the fastest estimate among the forms whose clusters all fit one
// wave (occupancy calculator) within `sms` CTAs.  {0, 0} when none does.
struct ClusterPick {
  int bn, splits;
};
ClusterPick pick_cluster_form(int64_t rows, int64_t n, int64_t k, int sms, int max_smem) {
  const int64_t m_blocks = (rows + BM - 1) / BM;
  ClusterPick best{0, 0};
  double best_t = 1e300;
  for (const Candidate &f : kClusterForms) {
    if (config_smem(f.bn, 0, kDenseCluster) > max_smem) continue;
    const int64_t tiles = m_blocks * ((n + f.bn - 1) / f.bn);
    for (int s = 2; s <= kMaxClusterSplits; ++s) {
      if (tiles * s > sms || s > k / BK) break;
      if (cluster_split_fit(f.bn, s) < tiles) continue;
      const double e = estimate_cluster(m_blocks, n, k, f, s);
      if (e < best_t * 0.99) {
        best_t = e;
        best = {f.bn, s};
      }
    }
  }
  return best;
}

size_t split_ws_bytes(int64_t tiles, int splits, int bn) {
  return static_cast<size_t>(tiles) * splits * BM * bn * 4 + tiles * 4;
}

struct Choice {
  int bn, splits;
  int64_t full_tiles;  // dense: tiles computed whole; the rest are split
};

// Estimated time of the dense "tail split": the whole waves of tiles, then
// the tiles of the last, partial wave split `s` ways along K over the CTAs.
double estimate_tail(int64_t waves, int64_t k, int bn, int s) {
  const int64_t kb = k / BK;
  const double whole = waves * (kb * kb_cycles(bn) + 2500.0);
  return whole + ((kb + s - 1) / s) * kb_cycles(bn) + 2500.0 + 1500.0 + 300.0 * s;
}

// Tile form for a launch: a tile width and K split from the cost model.
// Splitting every tile's K is considered for dense shapes of at most two M
// blocks, only while all units fit in one wave of CTAs; larger dense shapes
// may split only the tiles of a last, partial wave (spreading them over all
// CTAs).  Either needs a workspace that holds the split tiles' FP32 partials
// (`ws_bytes`).  Tile forms whose shared memory (with `extra` bytes of
// masked prefix tables) exceeds `max_smem` are skipped.
Choice choose_config(int sched, int64_t rows, int64_t n, int64_t k, int groups, int num_sms,
                     size_t ws_bytes, int extra = 0, int max_smem = 232448,
                     int layout = kLayoutNT) {
  const int64_t m_blocks = (rows + BM - 1) / BM;
  const int64_t k_blocks = k / BK;
  const int64_t m_blocks_eff =
      (sched == kMasked || sched == kKGrouped) ? m_blocks * groups : m_blocks;
  Choice c{128, 1, 0};
  double best = 1e300;
  for (const Candidate &cand : kCandidates) {
    if (config_smem(cand.bn, extra, sched) > max_smem) continue;
    // transposed layouts: whole 128-value MN-major columns of B
    if (layout != kLayoutNT && cand.bn % 128 != 0) continue;
    const int64_t tiles = m_blocks * ((n + cand.bn - 1) / cand.bn);
    for (int s = 1; s <= 16; ++s) {
      if (s > 1 && (sched != kDense || m_blocks > 2)) break;
      if (s > k_blocks) break;
      if (s > 1 && tiles * s > num_sms) break;
      if (s > 1 && split_ws_bytes(tiles, s, cand.bn) > ws_bytes) break;
      const double e = estimate(m_blocks_eff, n, k, cand.bn, s, num_sms);
      if (e < best * 0.97) {
        best = e;
        c = {cand.bn, s, 0};
      }
    }
    if (sched == kDense && m_blocks > 2) {
      const int64_t waves = tiles / num_sms, tail = tiles % num_sms;
      const int s = tail > 0 ? static_cast<int>(std::min<int64_t>(num_sms / tail, 16)) : 1;
      if (waves > 0 && s >= 2 && s <= k_blocks && split_ws_bytes(tail, s, cand.bn) <= ws_bytes) {
        const double bytes = static_cast<double>(n) * k + m_blocks * 128.0 * k;
        const double e = std::max(estimate_tail(waves, k, cand.bn, s), bytes / (23.0 * num_sms));
        if (e < best * 0.97) {
          best = e;
          c = {cand.bn, s, waves * num_sms};
        }
      }
    }
  }
  return c;
}

}  // namespace

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  // the split the heuristic picks when the workspace is not a constraint
  // the larger of the splits the NT layout and the transposed layouts (tiles
  // of 128 or 256 only) prefer
  size_t need = 0;
  for (int layout : {kLayoutNT, kLayoutTN}) {
    const Choice c = choose_config(kDense, M, N, K, 1, num_sms, ~static_cast<size_t>(0), 0,
                                   232448, layout);
    if (c.splits <= 1) continue;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + c.bn - 1) / c.bn) - c.full_tiles;
    need = std::max(need, split_ws_bytes(tiles, c.splits, c.bn));
  }
  return need == 0 ? 0 : (need + 255) & ~static_cast<size_t>(255);
}

// Test knobs of the abort path (both unset in normal use):
// DG_TEST_STARVE_LOAD=i makes CTA 0's producer leave out the loads of its
// iteration i (a kernel parameter); DG_TEST_WAIT_LIMIT_US=t lowers every
// wait's limit to t microseconds (at least kWaitCheckNs), written to the
// device before this call's kernel and put back after it, in stream order.
struct TestKnobs {
  int starve = -1;
  unsigned long long limit_ns = kWaitLimitNs;
};

static TestKnobs test_knobs() {
  TestKnobs k;
  if (const char *e = getenv("DG_TEST_STARVE_LOAD")) k.starve = atoi(e);
  if (const char *e = getenv("DG_TEST_WAIT_LIMIT_US"))
    k.limit_ns = strtoull(e, nullptr, 10) * 1000ull;
  return k;
}

static int set_wait_limit(unsigned long long limit_ns, cudaStream_t stream) {
  return cudaMemcpyToSymbolAsync(g_wait_limit_ns, &limit_ns, sizeof(limit_ns), 0,
                                 cudaMemcpyHostToDevice, stream) == cudaSuccess
             ? DG_OK
             : DG_ERR_CUDA;
}

static int launch_fp8_gemm_impl(int sched, const uint8_t *A, const uint8_t *B, GemmParams p,
                                cudaStream_t stream, int num_sms, size_t ws_bytes, void *ws,
                                int layout);

int launch_fp8_gemm(int sched, const uint8_t *A, const uint8_t *B, GemmParams p,
                    cudaStream_t stream, int num_sms, size_t ws_bytes, void *ws, int layout) {
  const TestKnobs knobs = test_knobs();
  p.starve_it = knobs.starve;
  if (knobs.limit_ns == kWaitLimitNs)
    return launch_fp8_gemm_impl(sched, A, B, p, stream, num_sms, ws_bytes, ws, layout);
  int rc = set_wait_limit(knobs.limit_ns, stream);
  if (rc) return rc;
  rc = launch_fp8_gemm_impl(sched, A, B, p, stream, num_sms, ws_bytes, ws, layout);
  const int rc2 = set_wait_limit(kWaitLimitNs, stream);
  return rc ? rc : rc2;
}

static int launch_fp8_gemm_impl(int sched, const uint8_t *A, const uint8_t *B, GemmParams p,
                                cudaStream_t stream, int num_sms, size_t ws_bytes, void *ws,
                                int layout) {
  const int64_t rows = p.rows, n = p.n, k = p.k;
  // transposed layouts: the plain dense GEMM (no C) and the k-grouped GEMM
  if (layout != kLayoutNT && !(sched == kKGrouped || (sched == kDense && p.c == nullptr)))
    return DG_ERR_INVALID_ARG;
  p.num_k_blocks = static_cast<int>(k / BK);
  if (ws == nullptr) ws_bytes = 0;

  // ------------------------------------------------ choose the tile form
  // masked launches keep per-expert row-block counts and prefix sums in
  // shared memory
  const int extra = base_sched(sched) == kMasked ? 8 * (p.groups + 1)
                    : sched == kKGrouped ? 4 * (p.groups + 1) : 0;
  const int max_smem = max_smem_per_block();
  if (is_ue8m0(sched)) {
    // one tile form, no K split: the whole tile sums K in TMEM
    if (config_smem(kUECandidate.bn, extra, sched) > max_smem) return DG_ERR_INVALID_ARG;
    const int bn = kUECandidate.bn;
    p.num_m_blocks = static_cast<int>((rows + BM - 1) / BM);
    p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
    p.splits = 1;
    p.full_tiles = 0;
    p.ws = nullptr;
    p.a_box_rows = BM;
    CUtensorMap ta, tb, td = {};
    const bool masked = base_sched(sched) == kMasked;
    int rc = make_tmap(&ta, A, k, rows, masked ? p.groups : 1, BM);
    if (rc) return rc;
    rc = make_tmap(&tb, B, k, n, masked ? p.groups : 1, bn);
    if (rc) return rc;
    if ((rc = make_tmap_d(&td, p.d, rows, n, masked ? p.groups : 1))) return rc;
    const int64_t units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks *
                          (masked ? p.groups : 1);
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
    if (print_configs())
      fprintf(stderr, "[dg] gemm sched=%d (UE8M0) rows=%lld n=%lld k=%lld groups=%d grid=%d\n",
              sched, static_cast<long long>(rows), static_cast<long long>(n),
              static_cast<long long>(k), p.groups, grid);
    return masked ? dispatch<kMaskedUE8M0>(bn, ta, tb, td, p, grid, extra, stream)
                  : dispatch<kDenseUE8M0>(bn, ta, tb, td, p, grid, extra, stream);
  }
  if (sched == kDenseQuant) {
    // whole 128-column groups per thread: 256-wide tiles, K never split (a
    // split tile's reduction spreads a row's group over several threads)
    const int bn = 256;
    p.num_m_blocks = static_cast<int>((rows + BM - 1) / BM);
    p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
    p.splits = 1;
    p.full_tiles = 0;
    p.ws = nullptr;
    p.a_box_rows = rows <= BM / 2 ? BM / 2 : BM;
    CUtensorMap ta, tb, td = {};
    int rc = make_tmap(&ta, A, k, rows, 1, p.a_box_rows);
    if (rc) return rc;
    rc = make_tmap(&tb, B, k, n, 1, bn);
    if (rc) return rc;
    const int64_t units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
    return dispatch<kDenseQuant>(bn, ta, tb, td, p, grid, extra, stream);
  }
  // The 2-CTA form for dense NT shapes of at least two M blocks: each SM
  // loads its 128 rows of A and half of the 256-wide B tile, two thirds of
  // the single-CTA form's operand bytes per K block.  DG_PAIR=1 / 0 forces
  // it on / off.
  bool pair = false;
  if (sched == kDense && p.c == nullptr && layout == kLayoutNT && rows > BM && n >= 256 &&
      num_sms >= 2) {
    pair = kPairByDefault;
    if (const char *e = getenv("DG_PAIR")) pair = *e == '1';
  }
  if (pair) {
    const int bn = 256;
    p.num_m_blocks = static_cast<int>((rows + 2 * BM - 1) / (2 * BM));
    p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
    p.splits = 1;
    p.full_tiles = 0;
    p.ws = nullptr;
    p.a_box_rows = BM;
    CUtensorMap ta, tb, td = {};
    int rc = make_tmap(&ta, A, k, rows, 1, BM);
    if (rc) return rc;
    rc = make_tmap(&tb, B, k, n, 1, bn / 2);
    if (rc) return rc;
    if ((rc = make_tmap_d(&td, p.d, rows, n, 1))) return rc;
    const int64_t units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
    const int grid =
        2 * static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms / 2)));
    if (print_configs())
      fprintf(stderr, "[dg] gemm sched=dense rows=%lld n=%lld k=%lld: 2-CTA BN=256 grid=%d\n",
              static_cast<long long>(rows), static_cast<long long>(n),
              static_cast<long long>(k), grid);
    return dispatch<kDensePair>(bn, ta, tb, td, p, grid, extra, stream);
  }
  const Choice choice =
      choose_config(sched, rows, n, k, p.groups, num_sms, ws_bytes, extra, max_smem, layout);
  int bn = choice.bn, splits = choice.splits;
  int64_t full_tiles = choice.full_tiles;
  bool splits_forced = false;  // DG_SPLITS: exactly this many, or none
  bool bn_forced = false;      // DG_BLOCK_N
  // D = C + A B^T (dense only): single-CTA tiles, splits through the
  // workspace (the FP32 tile is staged in the 32 KB the BF16 tile uses, so
  // every tile form still fits)
  const bool acc = p.c != nullptr;
  // Tuning / test overrides: DG_BLOCK_N forces the N tile, DG_SPLITS splits
  // every tile's K, DG_TAIL_SPLITS only the last partial wave's tiles (dense;
  // both need enough workspace).
  if (const char *e = getenv("DG_BLOCK_N")) {
    // (a non-power-of-two width serves the cluster split only: NT, with
    // DG_SPLITS of at least 2)
    const int v = atoi(e);
    bool known = false;
    for (const Candidate &c : kCandidates) known = known || c.bn == v;
    for (const Candidate &c : kClusterForms) known = known || (c.bn == v && layout == kLayoutNT);
    if (known && (layout == kLayoutNT || v % 128 == 0)) {
      if (v != bn) {
        bn = v;
        splits = 1;  // the split chosen for another width does not carry over
        full_tiles = 0;
      }
      bn_forced = true;
    }
  }
  if (const char *e = getenv("DG_SPLITS")) {
    // every tile split v ways (v = 1: no split)
    const int v = atoi(e);
    if (v >= 1) {
      const int64_t tiles = ((rows + BM - 1) / BM) * ((n + bn - 1) / bn);
      if (v > 1 && (sched != kDense || ws == nullptr || split_ws_bytes(tiles, v, bn) > ws_bytes ||
                    v > p.num_k_blocks))
        return DG_ERR_WORKSPACE;
      if (v > 1 && tiles * v > num_sms) return DG_ERR_INVALID_ARG;  // one unit per CTA
      splits = v;
      full_tiles = 0;
      splits_forced = true;
    }
  }
  if (const char *e = getenv("DG_TAIL_SPLITS")) {
    // the tiles of a partial last wave split v ways, after whole waves
    const int v = atoi(e);
    if (v >= 2 && sched == kDense) {
      const int64_t tiles = ((rows + BM - 1) / BM) * ((n + bn - 1) / bn);
      const int64_t waves = tiles / num_sms, tail = tiles % num_sms;
      if (waves == 0 || tail == 0 || tail * v > num_sms || v > p.num_k_blocks)
        return DG_ERR_INVALID_ARG;
      if (ws == nullptr || split_ws_bytes(tail, v, bn) > ws_bytes) return DG_ERR_WORKSPACE;
      splits = v;
      full_tiles = waves * num_sms;
    }
  }
  // (a non-power-of-two width exists only as the cluster split's form)
  const int smem_sched = (bn & (bn - 1)) != 0 ? kDenseCluster
                         : sched == kDense && acc ? kDenseAcc
                                                  : sched;
  if (config_smem(bn, extra, smem_sched) > max_smem) return DG_ERR_INVALID_ARG;  // too many experts
  p.num_m_blocks = static_cast<int>((rows + BM - 1) / BM);
  p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
  p.splits = splits;
  p.full_tiles = splits > 1 ? static_cast<int>(full_tiles) : 0;
  int64_t all_tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
  p.ws = nullptr;
  if (sched != kKGrouped) p.ws_ticket = nullptr;  // (k-grouped: ld_sfb shares it)
  // Every tile split (decode-sized shapes, one wave): the splits of a tile
  // form a cluster and reduce through distributed shared memory, needing no
  // workspace or arrival counters, when all clusters fit in one wave
  // (DG_CLUSTER_SPLIT=0 forces the workspace path).
  bool try_cluster = sched == kDense && !acc && splits > 1 && splits <= kMaxClusterSplits &&
                     p.full_tiles == 0 && all_tiles * splits <= num_sms;
  if (const char *e = getenv("DG_CLUSTER_SPLIT"))
    if (*e == '0') try_cluster = false;
  // ... with the width and split the bandwidth model prefers among the
  // cluster forms that fit one wave, non-power-of-two widths included
  // (unless DG_BLOCK_N / DG_SPLITS force them)
  bool picked = false;
  if (try_cluster && layout == kLayoutNT && !bn_forced && !splits_forced) {
    const ClusterPick cp = pick_cluster_form(rows, n, k, num_sms, max_smem);
    if (cp.bn > 0) {
      bn = cp.bn;
      splits = cp.splits;
      p.splits = splits;
      p.num_n_blocks = static_cast<int>((n + bn - 1) / bn);
      all_tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
      picked = true;
    }
  }
  // the workspace path: FP32 partials and one arrival counter per split tile
  auto setup_workspace = [&]() -> int {
    const int64_t split_tiles = all_tiles - p.full_tiles;
    if (ws == nullptr || split_ws_bytes(split_tiles, splits, bn) > ws_bytes)
      return DG_ERR_WORKSPACE;
    const size_t part = static_cast<size_t>(split_tiles) * splits * BM * bn * 4;
    p.ws = static_cast<float *>(ws);
    p.ws_ticket = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + part);
    if (cudaMemsetAsync(p.ws_ticket, 0, split_tiles * 4, stream) != cudaSuccess)
      return DG_ERR_CUDA;
    return DG_OK;
  };
  if (splits > 1 && !try_cluster) {
    const int rc = setup_workspace();
    if (rc) return rc;
  }

  // ------------------------------------------------ tensor maps
  CUtensorMap ta, tb, td = {};
  p.a_box_rows = (sched == kDense && rows <= BM / 2 && !a_mn_major(layout)) ? BM / 2 : BM;
  int rc = a_mn_major(layout)
               ? make_tmap_mn(&ta, A, rows, k, 1)
               : make_tmap(&ta, A, k, rows, sched == kMasked ? p.groups : 1, p.a_box_rows);
  if (rc) return rc;
  rc = b_mn_major(layout)
           ? make_tmap_mn(&tb, B, n, k, 1)
           : make_tmap(&tb, B, k, n, (sched == kDense || sched == kKGrouped) ? 1 : p.groups, bn);
  if (rc) return rc;
  // the plain dense tiles store D with TMA
  if (sched == kDense && !acc && (rc = make_tmap_d(&td, p.d, rows, n, 1))) return rc;

  // ------------------------------------------------ grid
  int64_t units;
  if (sched == kMasked) {
    // upper bound; the kernel reads the actual count from masked_m
    units = static_cast<int64_t>(p.num_m_blocks) * p.groups * p.num_n_blocks;
  } else if (sched == kKGrouped) {
    units = static_cast<int64_t>(p.groups) * all_tiles;
    if (units > 0x7FFFFFFF) return DG_ERR_INVALID_ARG;
  } else {
    units = p.full_tiles + (all_tiles - p.full_tiles) * splits;
  }
  int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
  if (try_cluster) {
    // the chosen split, else (unless forced) fewer splits while the grid
    // still keeps 3/5 of the SMs busy
    int rc = kClusterNoFit;
    const int chosen = p.splits;
    // (a picked form fits by construction: the launch asks the same cached
    // occupancy query)
    const int lowest = splits_forced || picked ? chosen : 2;
    for (int sc = chosen; sc >= lowest && rc == kClusterNoFit; --sc) {
      if (sc < chosen && all_tiles * sc * 5 < static_cast<int64_t>(num_sms) * 3) break;
      p.splits = sc;
      grid = static_cast<int>(all_tiles * sc);
      rc = layout == kLayoutNT
               ? dispatch<kDenseCluster>(bn, ta, tb, td, p, grid, extra, stream)
               : dispatch_any_layout<kDenseCluster>(layout, bn, ta, tb, td, p, grid, extra, stream);
    }
    if (rc == kClusterNoFit && picked) return DG_ERR_CUDA;  // (the query disagreed with itself)
    if (rc == kClusterNoFit) {
      p.splits = chosen;
      grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms)));
    }
    if (rc != kClusterNoFit) {
      if (print_configs())
        fprintf(stderr,
                "[dg] gemm sched=dense rows=%lld n=%lld k=%lld: single BN=%d splits=%d "
                "(cluster reduction) grid=%d\n",
                static_cast<long long>(rows), static_cast<long long>(n),
                static_cast<long long>(k), bn, p.splits, grid);
      return rc;
    }
    const int wrc = setup_workspace();  // the clusters do not fit one wave
    if (wrc) return wrc;
  }
  if (print_configs()) {
    fprintf(stderr,
            "[dg] gemm sched=%d rows=%lld n=%lld k=%lld groups=%d: BN=%d splits=%d "
            "whole=%d grid=%d units=%lld\n",
            sched, static_cast<long long>(rows), static_cast<long long>(n),
            static_cast<long long>(k), p.groups, bn, splits,
            p.full_tiles, grid, static_cast<long long>(units));
  }
  switch (sched) {
    case kDense:
      if (layout != kLayoutNT)
        return dispatch_any_layout<kDense>(layout, bn, ta, tb, td, p, grid, extra, stream);
      return acc ? dispatch<kDenseAcc>(bn, ta, tb, td, p, grid, extra, stream)
                 : dispatch<kDense>(bn, ta, tb, td, p, grid, extra, stream);
    case kContiguous: return dispatch<kContiguous>(bn, ta, tb, td, p, grid, extra, stream);
    case kMasked: return dispatch<kMasked>(bn, ta, tb, td, p, grid, extra, stream);
    case kKGrouped:
      // the k-grouped form's transposed variant is TN (both operands stored
      // with the token axis K outermost)
      if (layout == kLayoutTN)
        return dispatch_layout<kKGrouped, kLayoutTN>(bn, ta, tb, td, p, grid, extra, stream);
      if (layout != kLayoutNT) return DG_ERR_INVALID_ARG;
      return dispatch<kKGrouped>(bn, ta, tb, td, p, grid, extra, stream);
    default: return DG_ERR_INVALID_ARG;
  }
}

}  // namespace dg
