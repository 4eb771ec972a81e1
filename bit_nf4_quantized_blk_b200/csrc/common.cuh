// Shared device helpers of the QLoRA NF4 library (sm_100a only).
//
// PTX wrappers for shared-memory barriers, TMA tensor copies, the fifth
// generation tensor cores (tcgen05) and their tensor memory, plus the status
// word every kernel reports device-side errors to.  Every spin on a barrier is
// bounded in time: on expiry the waiting thread records QLORA_ERR_TIMEOUT,
// raises the CTA's abort flag and returns false, so no kernel can hang.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/qlora_nf4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace qnf4 {

constexpr int kBlock = 64;         // weights per first-level block
constexpr int kDqBlock = 256;      // first-level scales per double-quant chunk
constexpr int kChunkWeights = kBlock * kDqBlock;  // 16384 weights per chunk
constexpr int kMaxRank = 64;       // largest LoRA rank the kernels take
constexpr int kRankPad = 64;       // padded row length of rank-r side buffers

// Workspace header: the first 256 bytes of every workspace hold the device
// status word (sticky error code); the host carves the rest after it.
constexpr size_t kWsHeader = 256;

// Time limit of every device-side wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// ---------------------------------------------------------------------------
// Generic helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Record a device error in the status word (first error wins).
__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Debug-build checks.  A library built with -DQLORA_CHECKS
// (libqlora_nf4_checks.so, `build(checks=True)`) tests index and alignment
// conditions before the accesses they guard: a failed test records
// QLORA_ERR_CHECK in the call's status word (when it has one) and the access
// is skipped, with no trap; a skipped tensor copy then ends its consumer's
// bounded wait.  In the default build every test is the constant true and
// compiles away.
#ifdef QLORA_CHECKS
constexpr bool kChecks = true;
#else
constexpr bool kChecks = false;
#endif

__device__ __forceinline__ bool qlora_checked(int* status, bool ok) {
  if (kChecks && !ok) raise_status(status, QLORA_ERR_CHECK);
  return !kChecks || ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  // cvt.rn.bf16x2.f32 d, a, b packs a into the upper and b into the lower half.
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// 256-bit streaming load of 8 fp32 (read once: no L1 allocation).
__device__ __forceinline__ void ld_stream_v8(const float* p, float (&v)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "l"(p));
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 256-bit streaming store (one full 32-byte sector per lane).
__device__ __forceinline__ void st_stream_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void st_stream_u4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------------------
// mbarrier (shared-memory transaction barrier)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that also acquires what other CTAs of the cluster released.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase of parity `parity` of `bar` has completed.  Gives up
// after kWaitLimitNs or as soon as another thread of the CTA raised `abort`;
// on a timeout it records QLORA_ERR_TIMEOUT and raises `abort` itself.
// The abort flag and the clock are looked at once per 32 failed tries, so a
// waiting warp spends its issue slots on the barrier, not on the bookkeeping.
// `limit_ns` overrides the time limit (a diagnostic launch shortens it).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      raise_status(status, QLORA_ERR_TIMEOUT);
      return false;
    }
  }
}

// try_wait that may suspend the thread for up to `hint_ns` (it resumes as soon
// as the phase completes): a waiting warp then takes no issue slots.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, bool cluster, uint32_t hint_ns) {
  uint32_t ok;
  if (cluster)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
  return ok != 0;
}

// mbar_wait / mbar_wait_cluster for a thread whose wait is long and whose
// scheduler is shared with latency-critical work: each try may suspend it.
__device__ __forceinline__ bool mbar_wait_suspend(uint64_t* bar, uint32_t parity, bool cluster,
                                                  volatile int* abort_flag, int* status,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  constexpr uint32_t kHintNs = 2000;
  if (mbar_try_wait_suspend(bar, parity, cluster, kHintNs)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, cluster, kHintNs)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      raise_status(status, QLORA_ERR_TIMEOUT);
      return false;
    }
  }
}

// Same, ignoring the abort flag (teardown waits for work already in flight).
// Always the full limit: copies and MMAs already issued land within it.
__device__ __forceinline__ bool mbar_wait_teardown(uint64_t* bar, uint32_t parity, int* status) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, QLORA_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies; never with cluster multicast)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2-D tiled load global -> shared; completion is signalled on `bar` as bytes.
// Coordinates are in elements of kElemBytes bytes: c0 along the contiguous
// dimension (c0 * kElemBytes must be a multiple of 16; a checks build tests
// it and skips a copy that breaks it), c1 along rows.
template <int kElemBytes = 2>
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int* check_status = nullptr) {
  if (!qlora_checked(check_status, (c0 * kElemBytes) % 16 == 0)) return;
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 2-D tiled load into this CTA's shared memory whose completion (transaction
// bytes) is signalled on an mbarrier of either CTA of the pair, given by its
// shared::cluster address.  No multicast.
template <int kElemBytes = 2>
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 int c0, int c1, int* check_status = nullptr) {
  if (!qlora_checked(check_status, (c0 * kElemBytes) % 16 == 0)) return;
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
      : "memory");
}

// 1-D bulk copy global -> shared of `bytes` (multiple of 16; both addresses
// 16-byte aligned); completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the fifth-generation MMA
// ---------------------------------------------------------------------------

// Allocate `ncols` TMEM columns (power of two >= 32); the base address is
// written to shared memory at `dst`.  Executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void tc_mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every previously issued tcgen05.mma of this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (cluster of 2): the pair-CTA tensor-core MMA and its signals
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_cta(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on an mbarrier of the cluster (another CTA's, by its mapped address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Arrive on an mbarrier of the cluster with the instruction's default
// semantics (release at CTA scope).  For a signal whose consumer reads this
// CTA's shared memory only through the tensor core (async proxy): every
// writing thread has already ordered its writes for the async proxy with
// fence.proxy.async, and the MMA is issued after the other CTA's wait on this
// barrier.  A cluster-scope release here costs about 1,800 cycles per arrive
// on a B200 (it waits for the warp's memory operations to become visible
// cluster-wide), which made it the decoders' largest cost per stage.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bounded wait on a local barrier arrived at by the other CTA of the pair.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int* status, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      raise_status(status, QLORA_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Tensor memory of a CTA pair: executed by the same warp in both CTAs.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMA, issued by one thread of the even CTA: A rows 0..127 and B rows
// (N) 0..N/2-1 come from this CTA's shared memory, the other halves from the
// same offsets in the odd CTA's; each CTA's tensor memory receives its 128
// rows of D.
__device__ __forceinline__ void tc_mma_bf16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` (same offset) in every CTA of `cta_mask` once the pair
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"(cta_mask)
               : "memory");
}

// Load 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Load 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored in the
// 128-byte swizzle layout (rows of 64 bf16 = 128 bytes, 8-row atoms of 1024
// bytes, atoms stacked every 1024 bytes).  Bits: start address >> 4 at [0,14),
// leading byte offset >> 4 at [16,30) (unused for this layout, set to 1),
// stride byte offset >> 4 at [32,46), descriptor version 1 at [46,48),
// base offset 0, swizzle mode 2 (128B) at [61,64).
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Shared-memory matrix descriptor of an MN-major operand tile in the 128-byte
// swizzle layout: atoms of 8 rows along K x 128 bytes (64 bf16) along MN;
// `lbo` = byte stride between 64-element MN groups, `sbo` = byte stride
// between 8-row K groups.
__device__ __forceinline__ uint64_t smem_desc_mn128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator,
// A K-major, B K-major (b_mn = false) or MN-major (b_mn = true), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn = false) {
  return (1u << 4)                                  // D format: fp32
         | (1u << 7)                                // A format: bf16
         | (1u << 10)                               // B format: bf16
         | (b_mn ? (1u << 16) : 0u)                 // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------------------
// Warp-level legacy MMA (used by the HBM-bound skinny kernels and the GEMV,
// where the tensor pipe is far from the bound).
// ---------------------------------------------------------------------------

// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}

__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc, bool valid) {
  const int n = valid ? 16 : 0;  // src-size 0 writes zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(n)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: let the next kernel of the stream start its
// independent prologue / wait for the previous kernel's results.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// m16n8k16 bf16 MMA (warp-synchronous legacy tensor path), fp32 accumulate,
// d += a b.  Fragments (g = lane / 4, t = lane % 4; low half of a register =
// lower k): a0 (row g, k 2t..2t+1), a1 (row g+8, same k), a2 (row g,
// k 2t+8..2t+9), a3 (row g+8, same k); b0 (k 2t..2t+1, col g), b1 (k 2t+8..
// 2t+9, col g); d0, d1 (row g, cols 2t, 2t+1), d2, d3 (row g+8, same cols).
// Not `volatile`, so loads can be scheduled around it.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ---------------------------------------------------------------------------
// The NF4 codebook: the 16 levels of "QLoRA: NF4 storage, gradients and local
// integration", section "Exact CPU teaching quantizer and adapter gradient
// path" (exact fp32 values).
// ---------------------------------------------------------------------------
__host__ __device__ constexpr float nf4_level(int j) {
  return j == 0    ? -1.0f
         : j == 1  ? -0.6961928009986877f
         : j == 2  ? -0.5250730514526367f
         : j == 3  ? -0.39491748809814453f
         : j == 4  ? -0.28444138169288635f
         : j == 5  ? -0.18477343022823334f
         : j == 6  ? -0.09105003625154495f
         : j == 7  ? 0.0f
         : j == 8  ? 0.07958029955625534f
         : j == 9  ? 0.16093020141124725f
         : j == 10 ? 0.24611230194568634f
         : j == 11 ? 0.33791524171829224f
         : j == 12 ? 0.44070982933044434f
         : j == 13 ? 0.5626170039176941f
         : j == 14 ? 0.7229568362236023f
                   : 1.0f;
}

// The FP4 (E2M1) codebook of "FT-02: QLoRA -- Fine-Tuning with
// Quantization", section "Exercise 3: NF4 vs FP4 at equal memory": codes 0..7
// are the magnitudes k / 12, k = 0, 1/16, 2, 3, 4, 6, 8, 12 (printed there as
// 0, 0.0052, 0.1667, 0.25, 0.3333, 0.5, 0.6667, 1), rounded to fp32; code
// 8 + c is the negative of code c (bit 3 is the sign).
__host__ __device__ constexpr float fp4_level(int j) {
  return (j & 8 ? -1.0f : 1.0f) * ((j & 7) == 0   ? 0.0f
                                   : (j & 7) == 1 ? 0.005208333333333333f
                                   : (j & 7) == 2 ? 0.16666666666666666f
                                   : (j & 7) == 3 ? 0.25f
                                   : (j & 7) == 4 ? 0.3333333333333333f
                                   : (j & 7) == 5 ? 0.5f
                                   : (j & 7) == 6 ? 0.6666666666666666f
                                                  : 1.0f);
}

// Level j of a codebook (QLORA_CODEBOOK_NF4 or QLORA_CODEBOOK_FP4).
__host__ __device__ constexpr float codebook_level(int codebook, int j) {
  return codebook == QLORA_CODEBOOK_FP4 ? fp4_level(j) : nf4_level(j);
}

// Decision table of the nearest-level search on x in [-1, 1] (built once per
// codebook on the host, see api.cu).  A cell covers a fixed interval of x
// holding at most one decision threshold; pos(x) = base[c] + (x >= thr[c])
// (thr[c] = 4 where the cell holds none) is x's position among the
// codebook's distinct levels in increasing order.
//   NF4: cell c = trunc(64 x) + 64 (c = 0 .. 128); positions are the codes.
//   FP4: cell c = floor(64 x) + 65 (c = 0 .. 129; cells 0 and 129 catch
//        |64 x| a rounding past 64); positions 0 .. 14 over the 15 distinct
//        values (-0 is never chosen), mapped to codes by fp4_codes_of.
constexpr int kDecisionCells = 130;
struct Nf4DecisionTable {
  float thr[kDecisionCells];
  int base[kDecisionCells];
};

// Eight FP4 positions (nibbles, 0 .. 14) -> their sign-magnitude codes:
// positions 7 .. 14 are +0 .. +1 (codes 0 .. 7), positions 0 .. 6 are
// -1 .. -1/192 (codes 15 .. 9).  Nibble-parallel: first p16 = p + (p >= 7)
// (the 16-entry order with -0 at 7), then p16 >= 8 -> p16 - 8 and
// p16 < 8 -> 15 - p16, i.e. p16 ^ 8 ^ (p16 < 8 ? 7 : 0).  No nibble carries:
// p + 1 <= 15.
__host__ __device__ __forceinline__ uint32_t fp4_codes_of(uint32_t pos) {
  const uint32_t ge7 = ((pos + 0x11111111u) >> 3) & 0x11111111u;
  const uint32_t p16 = pos + ge7;
  const uint32_t lt8 = (~p16 >> 3) & 0x11111111u;
  return p16 ^ 0x88888888u ^ (lt8 * 7u);
}

__host__ __device__ __forceinline__ int fp4_code_of_position(int pos) {
  return static_cast<int>(fp4_codes_of(static_cast<uint32_t>(pos)) & 0xFu);
}

// Scale formats of a quantized tensor (qlora_scale_format).
constexpr int kScalesDqInt8 = QLORA_SCALES_DQ_INT8;
constexpr int kScalesDqFp8 = QLORA_SCALES_DQ_FP8;
constexpr int kScalesFp32 = QLORA_SCALES_FP32;

// E4M3 code -> fp32, exact: (1 + m/8) 2^(e-7) for e >= 1 (the fp32 bit
// pattern with exponent field e + 120 and the top mantissa bits m), m 2^-9
// for e = 0.  Stored scale codes are finite (never 0x7F / 0xFF).
__host__ __device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xFu, m = code & 7u;
  float v;
  if (e != 0) {
    const uint32_t bits = ((e + 120u) << 23) | (m << 20);
#ifdef __CUDA_ARCH__
    v = __uint_as_float(bits);
#else
    __builtin_memcpy(&v, &bits, 4);
#endif
  } else {
    v = static_cast<float>(m) * 0x1p-9f;
  }
  return (code & 0x80u) ? -v : v;
}

// The first factor of a double-quantized scale: fp32(q / 127) for int8
// codes, the E4M3 value for FP8 codes.
__device__ __forceinline__ float scale_code_value(int format, int8_t q) {
  return format == kScalesDqFp8 ? e4m3_to_float(static_cast<uint8_t>(q)) : __fdiv_rn(static_cast<float>(q), 127.0f);
}

// Decoded first-level scale: a = fp32(fp32(t * c2) + mu), t as above; two
// rounded operations in this order (no contraction into an FMA).
__device__ __forceinline__ float decode_scale_value(float t, float c2, float mu) {
  return __fadd_rn(__fmul_rn(t, c2), mu);
}

__device__ __forceinline__ float decode_scale(int q, float c2, float mu) {
  return decode_scale_value(__fdiv_rn(static_cast<float>(q), 127.0f), c2, mu);
}

}  // namespace qnf4
