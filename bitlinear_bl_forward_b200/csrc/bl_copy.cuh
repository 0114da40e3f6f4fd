// Copy of a host-buffer run between device-accessible pinned host memory and
// device memory, as a kernel rather than a copy-engine transfer: for the few
// kilobytes of a one-token step the copy engine's fixed latency is several
// times the transfer, while a kernel's loads and stores reach mapped pinned
// memory directly.
#pragma once

#include "bl_common.cuh"

namespace bl {

// 16-byte words across the grid, the last bytes % 16 by one thread (src and
// dst 16-byte aligned).  Ordered after the preceding kernel of the stream
// (programmatic dependent launch), and lets the next one start early.
__global__ void __launch_bounds__(256) bl_copy_run_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                                          size_t bytes) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n16 = bytes >> 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  if (blockIdx.x == 0 && threadIdx.x == 0)
    for (size_t b = n16 << 4; b < bytes; ++b) dst[b] = src[b];
}

}  // namespace bl
