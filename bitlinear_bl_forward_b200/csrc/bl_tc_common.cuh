// Constants shared by the tensor-core GEMMs (tile geometry), the identifiers
// of the pipeline waits a timeout records, and the self-test of the bounded
// wait.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kTcRows = 128;      // weight rows of one MMA tile (the MMA's M)
constexpr int kTcBK = 128;        // K of one 128-byte token box

// wait-site identifiers recorded with a timeout
enum : unsigned int {
  kSiteProdEmpty = 1,
  kSiteExpFull = 2,
  kSiteExpEmpty = 3,
  kSiteMmaExfull = 4,
  kSiteAcc = 5,
  kSiteDrain = 6,
  kSiteProbe = 7,
  kSiteSelftest = 0xEE
};

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives at; the wait must give up after limit_ns and record a timeout.
__global__ void bl_wait_selftest_kernel(unsigned long long limit_ns, int* out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const bool ok = mbar_wait(&bar, 0, nullptr, limit_ns, kSiteSelftest);
    *out = ok ? 1 : 0;
    // complete the phase so the barrier is not left pending
    mbar_arrive(&bar);
  }
}

}  // namespace bl
