// Decode path: ternary GEMV for one or two tokens, HBM-bound on the packed
// weights.
//
// "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear", eq. (3): Y = (X~ . W~^T) *
// (gamma / scale_X); section "Why 1.58 Bits? The Power of Zero": a weight adds,
// subtracts or skips the activation.  The products here are integer dot
// products of stored codes u = c + 1 in {0, 1, 2} with the int8 activations
// (__dp4a); sum_k c*q = sum_k u*q - sum_k q, and R = sum_k q is formed in the
// prologue.
//
// Structure (one kernel, fused activation quantisation):
//   1. every thread issues 128-bit loads for the first packed-weight chunks of
//      its first row tile (kept in registers) -- the HBM latency overlaps the
//      prologue;
//   2. prologue: the CTA quantises the MT token rows into shared memory
//      (per-token absmax, fp32 scale, round-half-even), in a layout whose
//      16-byte units are XOR-swizzled so the lanes of a warp read distinct
//      banks;
//   3. each warp owns RT output rows at a time; lane l takes the 64-weight
//      chunks l, l+32, ... of those rows, unpacks each 32-bit word with
//      shift+mask into four int8x4 lanes and accumulates with __dp4a;
//   4. warp-shuffle reduction, then offset correction and the fp32 rescale
//      (or the raw int32 accumulator) straight to global memory.
#pragma once

#include <cuda_bf16.h>

#include "bl_act.cuh"
#include "bl_common.cuh"

namespace bl {

enum OutMode : int { kOutBF16 = 0, kOutF32 = 1, kOutI32 = 2 };

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvPrefetch = 4;   // 64-weight chunks per lane prefetched per row

// Byte offset of activation byte kb of a token row inside the swizzled
// shared-memory copy: 128-byte lines, the 16-byte unit index XORed with the
// line index (low two bits).
__device__ __forceinline__ uint32_t act_swz(uint32_t kb) {
  const uint32_t line = kb >> 7, unit = (kb >> 4) & 7u;
  return (line << 7) | ((unit ^ (line & 3u)) << 4) | (kb & 15u);
}

__device__ __forceinline__ int block_reduce_max_f(float v, float* scratch) {
  // returns via scratch[0]; all threads must call
  v = warp_max(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = lane < kGemvWarps ? scratch[lane] : 0.f;
    t = warp_max(t);
    if (lane == 0) scratch[0] = t;
  }
  __syncthreads();
  return 0;
}

__device__ __forceinline__ int block_reduce_sum_i(int v, int* scratch) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kGemvWarps; ++w) t += scratch[w];
  return t;
}

template <int MT, int RT>
__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_kernel(const void* __restrict__ X, int x_is_i8, int M, int K, int N, const uint4* __restrict__ Wp,
                const float* __restrict__ gamma_p, int Q, void* __restrict__ Y, int out_mode) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_scale[MT];
  __shared__ float s_f[MT];
  __shared__ int s_R[MT];
  __shared__ float red_f[kGemvWarps];
  __shared__ int red_i[kGemvWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KV = K >> 6;                       // 64-weight (16-byte) chunks per row
  const uint32_t KL = ((K + 127) >> 7) << 7;   // bytes per token row in smem
  const int ntiles = (N + RT - 1) / RT;
  const int tstride = gridDim.x * kGemvWarps;
  int tile = blockIdx.x * kGemvWarps + warp;

  // 1. prefetch the first chunks of the first tile
  uint4 pw[kGemvPrefetch][RT];
#pragma unroll
  for (int u = 0; u < kGemvPrefetch; ++u)
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int c = lane + 32 * u, n = tile * RT + r;
      pw[u][r] = (tile < ntiles && c < KV && n < N) ? ldg_stream_v4(Wp + static_cast<size_t>(n) * KV + c)
                                                     : make_uint4(0, 0, 0, 0);
    }

  // 2. prologue: quantise the MT token rows into shared memory
  const uint32_t act_base = smem_u32(smem);
  for (int m = 0; m < MT; ++m) {
    int rsum = 0;
    if (!x_is_i8) {
      const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + static_cast<size_t>(m) * K);
      const int nch = K >> 3;
      float amax = 0.f;
      for (int c = threadIdx.x; c < nch; c += kGemvThreads) amax = fmaxf(amax, absmax8_bf16(__ldg(xr + c)));
      block_reduce_max_f(amax, red_f);
      const float s = __fdiv_rn(static_cast<float>(Q), fmaxf(red_f[0], 1e-5f));
      for (int c = threadIdx.x; c < nch; c += kGemvThreads) {
        const uint2 q = quant8_bf16(__ldg(xr + c), s, Q, rsum);
        const uint32_t off = m * KL + act_swz(static_cast<uint32_t>(c) << 3);
        *reinterpret_cast<uint2*>(smem + off) = q;
      }
      if (threadIdx.x == 0) {
        s_scale[m] = s;
        s_f[m] = (out_mode == kOutI32) ? 0.f : __fdiv_rn(*gamma_p, s);
      }
    } else {
      const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const int8_t*>(X) + static_cast<size_t>(m) * K);
      for (int c = threadIdx.x; c < (K >> 4); c += kGemvThreads) {
        const uint4 v = __ldg(xr + c);
        rsum = __dp4a(static_cast<int>(v.x), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.y), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.z), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.w), 0x01010101, rsum);
        *reinterpret_cast<uint4*>(smem + m * KL + act_swz(static_cast<uint32_t>(c) << 4)) = v;
      }
      if (threadIdx.x == 0) s_f[m] = 0.f;
    }
    const int tot = block_reduce_sum_i(rsum, red_i);
    if (threadIdx.x == 0) s_R[m] = tot;
  }
  __syncthreads();

  // 3. main loop over row tiles
  for (; tile < ntiles; tile += tstride) {
    int acc[RT][MT];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0;

    auto consume = [&](const uint4 (&w)[RT], int c) {
      // activation chunk c: 64 bytes = four 16-byte units of one 128-byte line
      uint4 a[MT][4];
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int g = 0; g < 4; ++g)
          a[m][g] = ld_shared_v4(act_base + m * KL + act_swz(static_cast<uint32_t>(c) * 64u + 16u * g));
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const uint32_t wd[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = static_cast<int>((wd[g] >> (2 * j)) & 0x03030303u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const uint32_t av[4] = {a[m][g].x, a[m][g].y, a[m][g].z, a[m][g].w};
              acc[r][m] = __dp4a(e, static_cast<int>(av[j]), acc[r][m]);
            }
          }
        }
      }
    };

#pragma unroll
    for (int u = 0; u < kGemvPrefetch; ++u) {
      const int c = lane + 32 * u;
      if (c < KV) consume(pw[u], c);
    }
    for (int c = lane + 32 * kGemvPrefetch; c < KV; c += 32) {
      uint4 w[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int n = tile * RT + r;
        w[r] = (n < N) ? ldg_stream_v4(Wp + static_cast<size_t>(n) * KV + c) : make_uint4(0, 0, 0, 0);
      }
      consume(w, c);
    }

    // prefetch the next tile before reducing this one
    const int nt = tile + tstride;
#pragma unroll
    for (int u = 0; u < kGemvPrefetch; ++u)
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int c = lane + 32 * u, n = nt * RT + r;
        pw[u][r] = (nt < ntiles && c < KV && n < N) ? ldg_stream_v4(Wp + static_cast<size_t>(n) * KV + c)
                                                     : make_uint4(0, 0, 0, 0);
      }

    // 4. reduce across the warp and write
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = warp_sum(acc[r][m]);
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int n = tile * RT + r;
        if (lane == r * MT + m && n < N && m < M) {
          const int a = acc[r][m] - s_R[m];
          const size_t o = static_cast<size_t>(m) * N + n;
          if (out_mode == kOutI32) {
            static_cast<int*>(Y)[o] = a;
          } else {
            const float y = __fmul_rn(__int2float_rn(a), s_f[m]);
            if (out_mode == kOutF32)
              static_cast<float*>(Y)[o] = y;
            else
              static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
          }
        }
      }
  }
}

}  // namespace bl
