// Device-side helpers shared by the BitLinear kernels (sm_100a only).
//
//   * a library-wide device status word that kernels set instead of trapping;
//   * mbarrier operations with BOUNDED waits (every spin gives up after a time
//     limit, records BL_ERR_TIMEOUT in the status word and lets the kernel
//     unwind cleanly);
//   * TMA (cp.async.bulk.tensor) 2-D tile loads into this CTA's shared memory;
//   * tcgen05 wrappers: TMEM alloc/dealloc, MMA kind::i8 with A in TMEM,
//     commit, 32x32b loads/stores and the thread-sync fences.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libbitlinear targets sm_100a only"
#endif

namespace bl {

// ---------------------------------------------------------------------------
// Device status word.  0 = OK.  Otherwise the low byte is a bl_status code
// and bits 8..15 identify the wait site that gave up.
// ---------------------------------------------------------------------------
__device__ unsigned int g_status = 0;

constexpr unsigned int kStatusTimeout = 6;   // == BL_ERR_TIMEOUT

__device__ __forceinline__ void record_status(unsigned int code, unsigned int site) {
  atomicCAS(&g_status, 0u, (code & 0xffu) | ((site & 0xffu) << 8));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
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

// Wait until the phase with the given parity has completed.  Returns false
// if another thread of the CTA raised *abort, or if limit_ns elapsed (then
// the status word records a timeout at `site` and *abort is raised so the
// rest of the CTA unwinds too).  abort may be null.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns,
                                          unsigned int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_status(kStatusTimeout, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// Cluster-scope variants for barriers that other CTAs of the cluster arrive
// on (the CTA pair of a cta_group::2 MMA).
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

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  uint64_t limit_ns, unsigned int site) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_status(kStatusTimeout, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// Arrive on the barrier at the same shared-memory offset in CTA `rank` of the
// cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

// Relaxed variant: for signalling completed tcgen05.st data (the data is in
// tensor memory once tcgen05.wait::st returns, and tcgen05.fence::before_
// thread_sync orders it before this arrive); a cluster-scope release here
// costs about half a microsecond per arrive.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA: 2-D tile load global -> shared, completion counted on an mbarrier.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory (addresses 16-byte
// aligned, size a multiple of 16), completion counted on an mbarrier.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier over `count` threads that also returns the AND of `v` over
// them, so the participants take the same decision.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// TMA 2-D tile store shared -> global (bulk-group completion), and the
// proxy fence that makes generic shared-memory writes visible to it.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tmap, int x, int y, const void* smem_src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
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
// All prior tcgen05 async ops of this thread arrive on the mbarrier when done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// CTA-pair (cta_group::2) forms: TMEM allocation in both CTAs, the MMA issued
// by the pair's leader, and a commit that arrives on the barrier at the same
// offset in every CTA named by cta_mask.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma_i8_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, int8 x int8 -> int32, cta_group::1.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Each thread of the warp writes 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: 8-row x 128-byte atoms, atoms 1024 bytes apart along the
// M/N dimension (stride byte offset), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);       // start address
  d |= static_cast<uint64_t>(1u) << 16;                          // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                  // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                          // version
  d |= static_cast<uint64_t>(2u) << 61;                          // SWIZZLE_128B
  return d;
}

// Sixteen tcgen05.mma kind::i8 (cta_group::2) of one K = 512 pipeline stage
// in one asm block.  MMA k (k = 0..15) reads A at tensor-memory column
// a0 + 8k and B through the shared-memory descriptor {dlo + boff(k), dhi},
// boff(k) = (k / 4) * BOX16 + 2 (k % 4) in the 16-byte units of the
// descriptor's start-address field (the sum cannot carry out of it for
// shared-memory addresses); the first MMA accumulates when acc0 != 0, the
// others always.  The issuing thread does nothing else between the MMAs: its
// instruction count per MMA bounds the MMA rate.
template <int BOX16>
__device__ __forceinline__ void mma_i8_stage16_pair(uint32_t d_tmem, uint32_t a0, uint32_t dlo, uint32_t dhi, uint32_t idesc,
                                                uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 d;\n\t.reg .b32 a, lo;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.eq.b32 q, %5, %5;\n\t"
      "mov.b64 d, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], d, %4, p;\n\t"
      "add.u32 a, %1, 8;\n\t"
      "add.u32 lo, %2, %6;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 16;\n\t"
      "add.u32 lo, %2, %7;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 24;\n\t"
      "add.u32 lo, %2, %8;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 32;\n\t"
      "add.u32 lo, %2, %9;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 40;\n\t"
      "add.u32 lo, %2, %10;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 48;\n\t"
      "add.u32 lo, %2, %11;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 56;\n\t"
      "add.u32 lo, %2, %12;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 64;\n\t"
      "add.u32 lo, %2, %13;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 72;\n\t"
      "add.u32 lo, %2, %14;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 80;\n\t"
      "add.u32 lo, %2, %15;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 88;\n\t"
      "add.u32 lo, %2, %16;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 96;\n\t"
      "add.u32 lo, %2, %17;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 104;\n\t"
      "add.u32 lo, %2, %18;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 112;\n\t"
      "add.u32 lo, %2, %19;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 120;\n\t"
      "add.u32 lo, %2, %20;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [a], d, %4, q;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a0), "r"(dlo), "r"(dhi),
         "r"(idesc), "r"(acc0), "n"((1 / 4) * BOX16 + 2 * (1 % 4)),
         "n"((2 / 4) * BOX16 + 2 * (2 % 4)), "n"((3 / 4) * BOX16 + 2 * (3 % 4)), "n"((4 / 4) * BOX16 + 2 * (4 % 4)), "n"((5 / 4) * BOX16 + 2 * (5 % 4)),
         "n"((6 / 4) * BOX16 + 2 * (6 % 4)), "n"((7 / 4) * BOX16 + 2 * (7 % 4)), "n"((8 / 4) * BOX16 + 2 * (8 % 4)), "n"((9 / 4) * BOX16 + 2 * (9 % 4)),
         "n"((10 / 4) * BOX16 + 2 * (10 % 4)), "n"((11 / 4) * BOX16 + 2 * (11 % 4)), "n"((12 / 4) * BOX16 + 2 * (12 % 4)), "n"((13 / 4) * BOX16 + 2 * (13 % 4)),
         "n"((14 / 4) * BOX16 + 2 * (14 % 4)), "n"((15 / 4) * BOX16 + 2 * (15 % 4))
      : "memory");
}

// Sixteen tcgen05.mma kind::i8 (cta_group::1) of one K = 512 pipeline stage
// in one asm block.  MMA k (k = 0..15) reads A at tensor-memory column
// a0 + 8k and B through the shared-memory descriptor {dlo + boff(k), dhi},
// boff(k) = (k / 4) * BOX16 + 2 (k % 4) in the 16-byte units of the
// descriptor's start-address field (the sum cannot carry out of it for
// shared-memory addresses); the first MMA accumulates when acc0 != 0, the
// others always.  The issuing thread does nothing else between the MMAs: its
// instruction count per MMA bounds the MMA rate.
template <int BOX16>
__device__ __forceinline__ void mma_i8_stage16(uint32_t d_tmem, uint32_t a0, uint32_t dlo, uint32_t dhi, uint32_t idesc,
                                                uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 d;\n\t.reg .b32 a, lo;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.eq.b32 q, %5, %5;\n\t"
      "mov.b64 d, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], d, %4, p;\n\t"
      "add.u32 a, %1, 8;\n\t"
      "add.u32 lo, %2, %6;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 16;\n\t"
      "add.u32 lo, %2, %7;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 24;\n\t"
      "add.u32 lo, %2, %8;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 32;\n\t"
      "add.u32 lo, %2, %9;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 40;\n\t"
      "add.u32 lo, %2, %10;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 48;\n\t"
      "add.u32 lo, %2, %11;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 56;\n\t"
      "add.u32 lo, %2, %12;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 64;\n\t"
      "add.u32 lo, %2, %13;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 72;\n\t"
      "add.u32 lo, %2, %14;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 80;\n\t"
      "add.u32 lo, %2, %15;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 88;\n\t"
      "add.u32 lo, %2, %16;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 96;\n\t"
      "add.u32 lo, %2, %17;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 104;\n\t"
      "add.u32 lo, %2, %18;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 112;\n\t"
      "add.u32 lo, %2, %19;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "add.u32 a, %1, 120;\n\t"
      "add.u32 lo, %2, %20;\n\t"
      "mov.b64 d, {lo, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [a], d, %4, q;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a0), "r"(dlo), "r"(dhi),
         "r"(idesc), "r"(acc0), "n"((1 / 4) * BOX16 + 2 * (1 % 4)),
         "n"((2 / 4) * BOX16 + 2 * (2 % 4)), "n"((3 / 4) * BOX16 + 2 * (3 % 4)), "n"((4 / 4) * BOX16 + 2 * (4 % 4)), "n"((5 / 4) * BOX16 + 2 * (5 % 4)),
         "n"((6 / 4) * BOX16 + 2 * (6 % 4)), "n"((7 / 4) * BOX16 + 2 * (7 % 4)), "n"((8 / 4) * BOX16 + 2 * (8 % 4)), "n"((9 / 4) * BOX16 + 2 * (9 % 4)),
         "n"((10 / 4) * BOX16 + 2 * (10 % 4)), "n"((11 / 4) * BOX16 + 2 * (11 % 4)), "n"((12 / 4) * BOX16 + 2 * (12 % 4)), "n"((13 / 4) * BOX16 + 2 * (13 % 4)),
         "n"((14 / 4) * BOX16 + 2 * (14 % 4)), "n"((15 / 4) * BOX16 + 2 * (15 % 4))
      : "memory");
}

// The constant high word and the start-address low word of a 128-byte-swizzled
// K-major descriptor (smem_desc_k_sw128 split in two).
constexpr uint32_t kDescSw128Hi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_sw128_lo(uint32_t smem_addr) { return ((smem_addr >> 4) & 0x3FFFu) | (1u << 16); }

// Instruction descriptor: kind::i8, s8 x s8 -> s32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
  return (2u << 4)                                   // D format: s32
         | (1u << 7)                                 // A: signed 8-bit
         | (1u << 10)                                // B: signed 8-bit
         | (static_cast<uint32_t>(n >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);    // M / 16
}

// Bulk prefetch of a contiguous global range into L2 by the TMA unit
// (address and size multiples of 16 bytes).  Only a hint: it reads nothing
// into the SM, so it is safe before griddepcontrol.wait.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: allow the next kernel of the stream (if it
// was launched with programmatic serialization) to start, and wait for the
// previous kernel's completion and memory flush (a no-op without PDL).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Read-only 16-byte load that the compiler may not move: issued exactly where
// it is written (used to start weight loads ahead of a barrier).
__device__ __forceinline__ uint4 ldg_pinned_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace bl
