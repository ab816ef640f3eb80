// ptx.cuh -- thin inline-PTX wrappers for the sm_100a primitives the GEMM uses:
// mbarriers (with bounded waits), TMA tensor loads, and the tcgen05 family
// (TMEM allocation, MMA issue, commit, TMEM loads, fences).
//
// Every wait in this library is bounded: it gives up after g_wait_limit_ns of
// %globaltimer, records DG_ERR_TIMEOUT in the device status word and returns
// false so that the caller can leave its loop and let the CTA exit cleanly.
#pragma once

#include <cstdint>

#include "dg.h"

namespace dg {

// Records `code` in the device status word unless an earlier error is there.
__device__ __forceinline__ void record_status(int *status, int code) {
  atomicCAS(status, 0, code);
}

// Two seconds: far above any legitimate wait inside one kernel.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// The limit every bounded wait of a kernel compiled in this translation unit
// applies (one copy per translation unit).  Its host side may lower it for a
// test that starves a wait on purpose, so that the wait runs out quickly.
static __device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

// Waits shorter than this never read g_wait_limit_ns, so that the limit's
// global load (cold in every cache at a kernel's start) stays off the path of
// ordinary waits; a lowered limit is therefore never below it.
constexpr uint64_t kWaitCheckNs = 1000000ull;

// Whether a wait that has run for `elapsed` ns is past the limit.
__device__ __forceinline__ bool wait_expired(uint64_t elapsed) {
  return elapsed > kWaitCheckNs && elapsed > g_wait_limit_ns;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar,
                                                      uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false (and
// records DG_ERR_TIMEOUT in *status) after g_wait_limit_ns, or soon after
// *abort is set by another role of the CTA that already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort, int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (wait_expired(globaltimer() - t0)) {
      record_status(status, DG_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spins until *counter >= target (acquire).  Returns false, recording
// DG_ERR_TIMEOUT, after g_wait_limit_ns.
__device__ __forceinline__ bool wait_counter(const uint32_t *counter, uint32_t target,
                                             int *status) {
  if (ld_acquire_gpu(counter) >= target) return true;
  const uint64_t t0 = globaltimer();
  while (ld_acquire_gpu(counter) < target) {
    __nanosleep(64);
    if (wait_expired(globaltimer() - t0)) {
      record_status(status, DG_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// 3-D tiled TMA load into shared memory, completing on mbarrier `bar`.
// Coordinates are element indices, innermost first.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap,
                                            uint32_t bar, int32_t c0,
                                            int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// tma_load_3d for the CTA pair of a cta_group::2 MMA: the box lands in this
// CTA's shared memory and its bytes complete on the mbarrier at the
// cluster-window address `bar` (the even CTA's, which counts both CTAs'
// bytes).  No multicast.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void *tmap, uint32_t bar,
                                                 int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 3-D tiled TMA store of a shared-memory box to global memory (the box's
// part outside the tensor is not written), tracked by this thread's bulk
// async-group.  Coordinates as for tma_load_3d; none negative.
__device__ __forceinline__ void tma_store_3d(const void *tmap, uint32_t src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          tmap),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Closes this thread's current bulk async-group.
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until every committed bulk group of this thread has finished reading
// its shared-memory source (the source may then be overwritten).
__device__ __forceinline__ void bulk_wait_group_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 1-D bulk copy global -> shared, completing on mbarrier `bar`.  Both
// addresses 16-byte aligned, `bytes` a positive multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src,
                                          uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ------------------------------------------------------------------ PDL
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream is still
// running.  It does its set-up (barrier initialisation, TMEM allocation,
// descriptor prefetch) first and calls grid_dependency_wait() before touching
// global memory: that returns once the previous grid has completed and its
// memory operations are visible, so stream order holds as before.
// grid_launch_dependents() lets the next such kernel start early.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Asks for the box of a 3-D tensor map at the given coordinates (as for
// tma_load_3d) to be brought into L2: no destination, nothing to wait for.
__device__ __forceinline__ void tma_prefetch_3d(const void *tmap, int32_t c0, int32_t c1,
                                                int32_t c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(tmap),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// Asks for `bytes` of global memory at `src` to be brought into L2 (no
// destination, no completion to wait for).  src 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ shared
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b,
                                             uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ------------------------------------------------------------------ FP32x2
// a0 = x0 * s + a0 and a1 = x1 * s + a1: two fused multiply-adds with one
// rounding each (to nearest even, subnormals kept, as fmaf) in one packed
// f32x2 instruction, which halves the issue slots of the promotion.
__device__ __forceinline__ void ffma2(float &a0, float &a1, float x0, float x1,
                                      float s) {
  asm("{\n\t.reg .b64 d, x, y;\n\t"
      "mov.b64 d, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %4};\n\t"
      "fma.rn.f32x2 d, x, y, d;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(s));
}

// a0 = x0 * s0 + a0 and a1 = x1 * s1 + a1: as ffma2 with a scale per lane.
__device__ __forceinline__ void ffma2v(float &a0, float &a1, float x0, float x1,
                                       float s0, float s1) {
  asm("{\n\t.reg .b64 d, x, y;\n\t"
      "mov.b64 d, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %5};\n\t"
      "fma.rn.f32x2 d, x, y, d;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(s0), "f"(s1));
}

// ------------------------------------------------------------------ registers
// Warp-specialised register split: a warpgroup lowers (dec) or raises (inc)
// its per-thread register count.  All four warps of a warpgroup execute the
// same instruction; an inc waits until the registers it asks for have been
// released by dec's of other warpgroups, so the split must fit the block's
// launch allocation (threads x registers per thread at launch).
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ tcgen05
// Allocates `ncols` TMEM columns (power of two >= 32); the base address is
// written to shared memory at `dst`.  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          dst),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile(
      "tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4, one CTA.  `accumulate` = 0
// overwrites D.  Issued by a single thread.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc,
                                        uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, "
      "%8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
      "r"(z), "r"(z)
      : "memory");
}

// Arrives once on `bar` when all tcgen05 operations issued so far by this
// thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// TMEM -> registers, 32 lanes x 32 bits, N consecutive columns per thread.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t *r);

template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
      "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld<64>(uint32_t taddr, uint32_t *r) {
  tmem_ld<32>(taddr, r);
  tmem_ld<32>(taddr + 32, r + 32);
}

// Orders uses of registers written by tcgen05.ld after the preceding
// tcgen05.wait::ld: the compiler cannot hoist a use above this point because
// the registers are (nominally) redefined here.
template <int N>
__device__ __forceinline__ void reg_barrier(uint32_t *r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i])::"memory");
}

// ------------------------------------------------------------------ clusters
// The split-K cluster reduction: the CTAs of a thread-block cluster read each
// other's shared memory (distributed shared memory).

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of every CTA of the cluster (release / acquire: shared-memory
// writes before it are visible to the cluster's reads after it).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address in the cluster shared window of the same shared-memory offset in
// CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// 16 bytes from the cluster shared window (this or a peer CTA's memory).
__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ------------------------------------------------------------------ CTA pairs
// The 2-CTA form: the two CTAs of a cluster (ranks 0 and 1) compute a
// 256-row tile with cta_group::2 MMAs issued by rank 0; each CTA holds its
// own 128 rows of A and half of the B tile, and its own 128 accumulator rows
// in TMEM.

// Arrive on the mbarrier at a cluster-window address (the peer's) with
// release semantics at cluster scope: the peer's acquire then sees what this
// thread saw (the stage's data, which landed on this CTA's own barrier).
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   cluster_addr)
               : "memory");
}

// Arrive on an mbarrier given by its cluster-window address (possibly in the
// peer CTA), default semantics: the arrive follows this thread's completed
// TMEM reads, which tcgen05.wait::ld and tcgen05.fence::before_thread_sync
// order.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_acquire_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait with acquire semantics at cluster scope (for a barrier the peer
// CTA arrives on with mbar_arrive_release_cluster); bounded like mbar_wait.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int *abort, int *status) {
  if (mbar_try_wait_acquire_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_acquire_cluster(bar, parity)) return true;
    if (*abort) return false;
    if (wait_expired(globaltimer() - t0)) {
      record_status(status, DG_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T with M = 256: rows 0-127 of A and D in
// rank 0, rows 128-255 in rank 1; B split along N between the two CTAs'
// shared memory at the same offsets.  Issued by one thread of rank 0.
__device__ __forceinline__ void umma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, "
      "%8, %9, %10, %11, %12}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z),
      "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}

// Arrives once on this CTA's mbarrier `bar` when all tcgen05 operations issued
// so far by this thread (pair MMAs included) have completed.
__device__ __forceinline__ void umma_commit_pair_own(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Arrives once on the mbarrier at offset `bar` in both CTAs of the pair when
// all tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster."
      "b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// ------------------------------------------------------------------ UMMA descriptors
// Shared-memory matrix descriptor for a K-major operand tile whose rows are
// 128 bytes (one 128-wide FP8 K block), written by TMA with the 128-byte
// swizzle: 8-row groups of 1024 bytes (stride byte offset 1024), descriptor
// version 1 (sm_100), layout type 2 (128-byte swizzle).  The tile base must be
// 1024-byte aligned; advancing along K inside the 128-byte row is done by
// adding the byte offset to the start address.
__device__ __forceinline__ uint64_t smem_desc_k128_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);      // start address
  d |= static_cast<uint64_t>(1) << 16;                     // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;             // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                     // version
  d |= static_cast<uint64_t>(2) << 61;                     // 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor for an MN-major operand tile written by TMA
// with the 128-byte swizzle: each K row holds 128 bytes (128 FP8 values) of
// M or N, 8 consecutive K rows form a 1024-byte swizzle atom (stride byte
// offset 1024 between atoms along K), and a tile wider than 128 values is
// several such 128-wide columns `lbo` bytes apart (leading byte offset).
// Advancing along K by 32 rows adds 4096 bytes to the start address.  The
// tile base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);      // start address
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;   // leading byte offset
  d |= static_cast<uint64_t>(1024 >> 4) << 32;             // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                     // version
  d |= static_cast<uint64_t>(2) << 61;                     // 128-byte swizzle
  return d;
}

// Shared-memory descriptor of a no-swizzle K-major source whose rows are 16
// bytes, stored contiguously (8-row core matrices of 128 bytes, one after
// the other): the source of tcgen05.cp's 32x128b shape.  Stride byte offset
// = 128 (next 8 rows), leading byte offset 128 (unused: one 16-byte column),
// version 1, layout type 0 (no swizzle).  saddr 16-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_rows16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);      // start address
  d |= static_cast<uint64_t>(128 >> 4) << 16;              // leading byte offset
  d |= static_cast<uint64_t>(128 >> 4) << 32;              // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                     // version
  return d;
}

// Instruction descriptor: kind::f8f6f4, A and B E4M3 (format 0), both
// K-major, FP32 accumulator (c_format 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int m, int n) {
  return (1u << 4) |                                // D format F32
         (0u << 7) | (0u << 10) |                   // A, B: E4M3
         (static_cast<uint32_t>(n >> 3) << 17) |    // N / 8
         (static_cast<uint32_t>(m >> 4) << 24);     // M / 16
}

// The same with the operands' majorness: bit 15 set when A is MN-major (its
// shared-memory tile holds K rows of M values), bit 16 when B is.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32_major(int m, int n, bool a_mn, bool b_mn) {
  return idesc_e4m3_f32(m, n) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
}

// Instruction descriptor of the block-scaled kind::mxf8f6f4: A and B E4M3
// (format 0), both K-major, UE8M0 scale factors (scale format 1 at bit 23),
// shape M x N; the FP32 accumulator is implied.  The byte of each 32-bit
// scale-factor cell to use (one of four K groups packed per cell) goes to
// bits 29-30 (A) and 4-5 (B), and to bits 30-31 of the scale-factor TMEM
// addresses given to the MMA.
__host__ __device__ constexpr uint32_t idesc_mxf8_ue8m0(int m, int n) {
  return (0u << 7) | (0u << 10) |                   // A, B: E4M3
         (static_cast<uint32_t>(n >> 3) << 17) |    // N / 8
         (1u << 23) |                               // scale factors UE8M0
         (static_cast<uint32_t>(m >> 4) << 24);     // M / 16
}

__host__ __device__ constexpr uint32_t idesc_sf_bytes(uint32_t idesc, uint32_t byte) {
  return idesc | (byte << 29) | (byte << 4);
}

// D[tmem] (+)= (A * 2^sfa) * (B * 2^sfb)^T, kind::mxf8f6f4 with one UE8M0
// scale factor per row of A and of B for the MMA's 32-wide K slice, read
// from TMEM at sfa_tmem / sfb_tmem (the byte within each cell in the top two
// address bits and in the instruction descriptor).  One thread issues.
__device__ __forceinline__ void umma_mxf8_ue8m0(uint32_t d_tmem, uint64_t a_desc,
                                                uint64_t b_desc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared memory -> TMEM: 32 rows of 128 bits (smem_desc_rows16 source) into
// 32 lanes x 4 columns at taddr, the same data written into each of the four
// 32-lane subpartitions (the replicated layout the block-scaled MMA reads
// its scale factors from).  Asynchronous; tcgen05 operations issued by the
// same thread after it (the MMAs that read these columns) see its result.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
               : "memory");
}

// 4-byte asynchronous copy global -> shared (both 4-byte aligned).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Arrives on `bar` (counting as one of its expected arrivals) once every
// cp.async this thread issued before has completed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

}  // namespace dg
