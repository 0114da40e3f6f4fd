// Throughput probe of the tensor-core instruction the prefill GEMMs use:
// tcgen05.mma kind::i8 (int8 x int8 -> int32), A in tensor memory, B in
// shared memory (128-byte swizzle), cta_group::1.  It measures the peak that
// the GEMMs' tensor-pipe fraction is quoted against.
//
// One CTA per SM; one thread issues `n_mma` MMAs of M = 128, N = n_cols,
// K = 32 back to back into one accumulator, then one commit; the CTA records
// the SM clock cycles and the global-timer nanoseconds from the first issue to
// the commit's completion.  The operands' contents do not matter (the MMA
// rate does not depend on the data), so shared and tensor memory are used as
// found.  The wait for the commit is bounded like every wait in the library.
#pragma once

#include "bl_tc_common.cuh"

namespace bl {

constexpr int kProbeThreads = 128;
constexpr int kProbeBBytes = 256 * 128;   // N <= 256 rows of 128 bytes (one swizzle atom column)
// more shared memory than the operand needs, so that no SM holds two CTAs
constexpr int kProbeSmemBytes = 128 * 1024 + 1024;

__device__ __forceinline__ uint64_t clock64_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
  return t;
}

// out[2 * blockIdx.x] = cycles, out[2 * blockIdx.x + 1] = nanoseconds.
__global__ void __launch_bounds__(kProbeThreads, 1)
    bl_probe_mma_i8_kernel(int n_mma, int n_cols, unsigned long long* __restrict__ out, unsigned long long limit_ns) {
  extern __shared__ uint8_t probe_raw[];
  uint8_t* sB = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(probe_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t done;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_i8(128, n_cols);
    const uint32_t b0 = smem_u32(sB);
    const uint32_t a_tmem = tmem + 256;   // 8 columns of A (128 lanes x 32 bytes)
    const uint64_t c0 = clock64_now();
    const uint64_t g0 = globaltimer_ns();
    for (int i = 0; i < n_mma; ++i)
      mma_i8_ts(tmem, a_tmem, smem_desc_k_sw128(b0 + 32 * (i & 3)), idesc, i != 0 ? 1u : 0u);
    tc_commit(&done);
    const bool ok = mbar_wait(&done, 0, nullptr, limit_ns, kSiteProbe);
    const uint64_t c1 = clock64_now();
    const uint64_t g1 = globaltimer_ns();
    out[2 * blockIdx.x] = ok ? (c1 - c0) : 0ull;
    out[2 * blockIdx.x + 1] = ok ? (g1 - g0) : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bl

namespace bl {

// The CTA-pair form (cta_group::2, a cluster of two CTAs, M = 256 split over
// the pair, N = n_cols with half of B in each CTA): the leader issues n_mma
// MMAs; both CTAs record cycles and nanoseconds to the commit's completion.
__global__ void __launch_bounds__(kProbeThreads, 1)
    bl_probe_mma_i8_pair_kernel(int n_mma, int n_cols, unsigned long long* __restrict__ out,
                                unsigned long long limit_ns) {
  extern __shared__ uint8_t probe_raw[];
  uint8_t* sB = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(probe_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t done;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_rank();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint64_t c0 = clock64_now();
  const uint64_t g0 = globaltimer_ns();
  if (threadIdx.x == 0 && rank == 0) {
    const uint32_t idesc = idesc_i8(256, n_cols);
    const uint32_t b0 = smem_u32(sB);
    const uint32_t a_tmem = tmem + 256;
    for (int i = 0; i < n_mma; ++i)
      mma_i8_ts_pair(tmem, a_tmem + 8 * (i & 3), smem_desc_k_sw128(b0 + 32 * (i & 3)), idesc, i != 0 ? 1u : 0u);
    tc_commit_pair(&done, 3);
  }
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait_cluster(&done, 0, nullptr, limit_ns, kSiteProbe);
  const uint64_t c1 = clock64_now();
  const uint64_t g1 = globaltimer_ns();
  if (threadIdx.x == 0) {
    out[2 * blockIdx.x] = ok ? (c1 - c0) : 0ull;
    out[2 * blockIdx.x + 1] = ok ? (g1 - g0) : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace bl
