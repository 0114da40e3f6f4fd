// Per-token absmax activation quantisation.
//
// "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear", eq. (2): scale_X = Q_b / (max_j |X_ij|
// + eps) per token, X~ = Round(Clip(X * scale_X, ...)).  Clip range [-128, 127]
// from "BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs", section "1. The
// BitLinear Operator"; the 4-bit mode (Q = 7, range [-8, 7]) from "BitNet a4.8
// Guide: 4-Bit Activation 1-Bit LLMs", section "1. Hybrid W1.58 / A4
// Quantization Function".  eps is read as a floor: s = Q / max(a, 1e-5).
//
// Every rounding is explicit so results are bit-identical to an IEEE fp32
// evaluation: __fdiv_rn for the scale, __fmul_rn for x * s (never fused),
// then round half to even to an integer.  That last step adds 1.5 * 2^23:
// for |v| < 2^22 the fp32 sum lies in [2^23, 2^24), where the spacing is 1,
// so the round-to-nearest-even addition leaves 1.5 * 2^23 + rint(v) (the
// constant is even, so ties go to even); |x * s| <= Q + 1 here.  Two
// full-rate instructions instead of a float-to-int conversion.
#pragma once

#include "bl_common.cuh"

namespace bl {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// max |x| of 8 bf16 as a pair of 16-bit magnitudes (non-negative bf16 bit
// patterns order like their values): accumulate with __vmaxu2, convert once
// with absmax2_f32.
__device__ __forceinline__ uint32_t absmax2_bf16x8(uint4 v) {
  constexpr uint32_t m = 0x7fff7fffu;
  return __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
}
__device__ __forceinline__ float absmax2_f32(uint32_t a2) { return __uint_as_float(max(a2 & 0xffffu, a2 >> 16) << 16); }
__device__ __forceinline__ float absmax8_bf16(uint4 v) { return absmax2_f32(absmax2_bf16x8(v)); }

// Four codes q = rint(x * s) (fp32 product, round half to even) as the bytes
// of one word.  x * s + 1.5 * 2^23 lies in [2^23, 2^24), where the spacing
// is 1, so its bit pattern is 0x4B400000 + rint(x * s) and its low byte is
// the code.  No clamp is needed: with a = max|x| and s = RN(Q / max(a, eps)),
// |x * s| <= Q (1 + 2^-24), whose fp32 rounding is at most one ulp above Q
// (Q = 7 or 127), so |q| <= Q and -Q-1 is never reached.
__device__ __forceinline__ uint32_t codes4(float a, float b, float c, float d, float s) {
  const uint32_t qa = __float_as_uint(__fadd_rn(__fmul_rn(a, s), 12582912.0f));
  const uint32_t qb = __float_as_uint(__fadd_rn(__fmul_rn(b, s), 12582912.0f));
  const uint32_t qc = __float_as_uint(__fadd_rn(__fmul_rn(c, s), 12582912.0f));
  const uint32_t qd = __float_as_uint(__fadd_rn(__fmul_rn(d, s), 12582912.0f));
  return __byte_perm(__byte_perm(qa, qb, 0x0040), __byte_perm(qc, qd, 0x0040), 0x5410);
}

// 8 bf16 -> 8 int8 codes (two 32-bit words), their sum added to `sum`.
__device__ __forceinline__ uint2 quant8_bf16(uint4 v, float s, int& sum) {
  const uint32_t lo = codes4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y), s);
  const uint32_t hi = codes4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w), s);
  sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
  return make_uint2(lo, hi);
}

// Input modes of the token prologues: bf16 activations, int8 codes given
// directly, the squared-ReLU feed-forward input ("BitNet 2B4T Guide:
// Scaling Native 1.58-Bit LLMs", section "2. Squared ReLU Activation"):
// h = max(0, g)^2 of the gate projection's bf16 output g, optionally times the
// up projection's output u, or bf16 activations RMS-normalised first (the
// same page, section "3. Sub-Layer Normalization (SubLN)") or
// layer-normalised first ("BitNet b1.58: The 1-Bit Ternary LLM Architecture
// Guide", BitLinear code listing).
enum InMode : int { kInBF16 = 0, kInI8 = 1, kInRelu2 = 2, kInRelu2Gated = 3, kInRmsNorm = 4, kInLayerNorm = 5 };

// h for 8 consecutive elements (fp32; exact for bf16 g and u).
__device__ __forceinline__ void relu2_8(uint4 g, uint4 u, bool gated, float (&h)[8]) {
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
  const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float r0 = fmaxf(bf16_lo(gw[i]), 0.f), r1 = fmaxf(bf16_hi(gw[i]), 0.f);
    h[2 * i] = __fmul_rn(r0, r0);
    h[2 * i + 1] = __fmul_rn(r1, r1);
    if (gated) {
      h[2 * i] = __fmul_rn(h[2 * i], bf16_lo(uw[i]));
      h[2 * i + 1] = __fmul_rn(h[2 * i + 1], bf16_hi(uw[i]));
    }
  }
}

__device__ __forceinline__ float absmax8_f32(const float (&h)[8]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(h[i]));
  return a;
}

// 8 fp32 values -> 8 codes (two 32-bit words), their sum added to `sum`.
__device__ __forceinline__ uint2 quant8_f32(const float (&h)[8], float s, int& sum) {
  const uint32_t lo = codes4(h[0], h[1], h[2], h[3], s), hi = codes4(h[4], h[5], h[6], h[7], s);
  sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kActRowsPerBlock = 8;   // one warp per token row
constexpr int kActCache = 16;         // 16-byte chunks kept in registers per lane

// X bf16 [M, K] -> Xq int8 [M, K], s[M] = Q / max(a, 1e-5), optional R[M] =
// sum_k Xq[m, k] (used to undo the +1 offset of the stored weight codes).
__global__ void __launch_bounds__(256) bl_act_quant_kernel(const uint16_t* __restrict__ X, int M, int K, int Q,
                                                        int8_t* __restrict__ Xq, float* __restrict__ s_out,
                                                        int* __restrict__ R_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * kActRowsPerBlock + warp;
  if (m >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K);
  const int nch = K >> 3;
  uint4 cache[kActCache];
  uint32_t a2 = 0u;
#pragma unroll
  for (int i = 0; i < kActCache; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      cache[i] = __ldg(xr + c);
      a2 = __vmaxu2(a2, absmax2_bf16x8(cache[i]));
    }
  }
  for (int c = lane + 32 * kActCache; c < nch; c += 32) a2 = __vmaxu2(a2, absmax2_bf16x8(__ldg(xr + c)));
  const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(absmax2_f32(a2))));
  const float s = __fdiv_rn(static_cast<float>(Q), fmaxf(amax, 1e-5f));
  uint2* qr = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(m) * K);
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kActCache; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) qr[c] = quant8_bf16(cache[i], s, sum);
  }
  for (int c = lane + 32 * kActCache; c < nch; c += 32) qr[c] = quant8_bf16(__ldg(xr + c), s, sum);
  sum = warp_sum(sum);
  if (lane == 0) {
    if (s_out) s_out[m] = s;
    if (R_out) R_out[m] = sum;
  }
}

// The same quantisation with one CTA per token row, for few rows: the
// absmax is a block reduction, so a row of K = 8192 costs four 16-byte loads
// a thread instead of 32 a lane.  Bit-identical to bl_act_quant_kernel (the max
// and the integer sum do not depend on the order).
constexpr int kActRowThreads = 256;
constexpr int kActRowCache = 8;   // 16-byte chunks kept in registers per thread (K <= 16384)

// Eight int8 codes in [-8, 7] (two words) -> eight two's-complement nibbles
// in one word: code 2j in the low nibble of byte j, code 2j + 1 in its high
// nibble.
__device__ __forceinline__ uint32_t pack_nibbles8(uint2 q) {
  const uint32_t lo = q.x & 0x0f0f0f0fu, hi = q.y & 0x0f0f0f0fu;
  const uint32_t a = lo | (lo >> 4), b = hi | (hi >> 4);   // bytes 0 and 2 hold code pairs
  return __byte_perm(a, b, 0x6420);
}

template <bool PACK4 = false>
__global__ void __launch_bounds__(kActRowThreads) bl_act_quant_row_kernel(const uint16_t* __restrict__ X, int K, int Q,
                                                                       int8_t* __restrict__ Xq,
                                                                       float* __restrict__ s_out,
                                                                       int* __restrict__ R_out,
                                                                       const uint32_t* __restrict__ amax_all) {
  constexpr int W = kActRowThreads / 32;
  __shared__ uint32_t s_max[W];
  __shared__ int s_sum[W];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const size_t m = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(X + m * K);
  const int nch = K >> 3;
  uint4 cache[kActRowCache];
  uint32_t a2 = 0u;
#pragma unroll
  for (int i = 0; i < kActRowCache; ++i) {
    const int c = t + kActRowThreads * i;
    if (c < nch) {
      cache[i] = __ldg(xr + c);
      a2 = __vmaxu2(a2, absmax2_bf16x8(cache[i]));
    }
  }
  for (int c = t + kActRowThreads * kActRowCache; c < nch; c += kActRowThreads)
    a2 = __vmaxu2(a2, absmax2_bf16x8(__ldg(xr + c)));
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(absmax2_f32(a2)));
  if (lane == 0) s_max[warp] = wmax;
  __syncthreads();
  uint32_t bmax = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) bmax = max(bmax, s_max[w]);
  if (amax_all) bmax = *amax_all;   // per-tensor mode: one absmax for every row
  const float s = __fdiv_rn(static_cast<float>(Q), fmaxf(__uint_as_float(bmax), 1e-5f));
  int sum = 0;
  if constexpr (PACK4) {
    // 4-bit codes, two a byte: row m is K / 2 bytes
    uint32_t* qr = reinterpret_cast<uint32_t*>(Xq + m * (K / 2));
#pragma unroll
    for (int i = 0; i < kActRowCache; ++i) {
      const int c = t + kActRowThreads * i;
      if (c < nch) qr[c] = pack_nibbles8(quant8_bf16(cache[i], s, sum));
    }
    for (int c = t + kActRowThreads * kActRowCache; c < nch; c += kActRowThreads)
      qr[c] = pack_nibbles8(quant8_bf16(__ldg(xr + c), s, sum));
  } else {
    uint2* qr = reinterpret_cast<uint2*>(Xq + m * K);
#pragma unroll
    for (int i = 0; i < kActRowCache; ++i) {
      const int c = t + kActRowThreads * i;
      if (c < nch) qr[c] = quant8_bf16(cache[i], s, sum);
    }
    for (int c = t + kActRowThreads * kActRowCache; c < nch; c += kActRowThreads)
      qr[c] = quant8_bf16(__ldg(xr + c), s, sum);
  }
  const int wsum = __reduce_add_sync(0xffffffffu, sum);
  if (lane == 0) s_sum[warp] = wsum;
  __syncthreads();
  if (t == 0) {
    int tot = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) tot += s_sum[w];
    if (s_out) s_out[m] = s;
    if (R_out) R_out[m] = tot;
  }
}

// Tensor-wide absmax of bf16 activations ("BitNet 2B4T Guide: Scaling Native
// 1.58-Bit LLMs", section "1. The BitLinear Operator", per-tensor form):
// non-negative floats order as their bit patterns, so a max of the bits is the
// max of the values.  *amax_out must be zero before the launch.
__global__ void __launch_bounds__(256) bl_act_absmax_kernel(const uint16_t* __restrict__ X, int64_t nchunks,
                                                        uint32_t* __restrict__ amax_out) {
  const uint4* x4 = reinterpret_cast<const uint4*>(X);
  float a = 0.f;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x)
    a = fmaxf(a, absmax8_bf16(__ldg(x4 + c)));
  const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_out, w);
}

// Squared-ReLU feed-forward input, quantised per token: one CTA per row;
// pass 1 takes the absmax of h over the row, pass 2 recomputes h (the row is
// in L1/L2 by then) and writes the codes.  G, U: bf16 [M, K] (U only when
// gated).
__global__ void __launch_bounds__(kActRowThreads) bl_act_quant_relu2_kernel(const uint16_t* __restrict__ G,
                                                                         const uint16_t* __restrict__ U, int gated,
                                                                         int K, int Q, int8_t* __restrict__ Xq,
                                                                         float* __restrict__ s_out,
                                                                         int* __restrict__ R_out) {
  constexpr int W = kActRowThreads / 32;
  __shared__ uint32_t s_max[W];
  __shared__ int s_sum[W];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const size_t m = blockIdx.x;
  const uint4* gr = reinterpret_cast<const uint4*>(G + m * K);
  const uint4* ur = gated ? reinterpret_cast<const uint4*>(U + m * K) : nullptr;
  const int nch = K >> 3;
  float amax = 0.f;
  for (int c = t; c < nch; c += kActRowThreads) {
    float h[8];
    relu2_8(__ldg(gr + c), gated ? __ldg(ur + c) : make_uint4(0, 0, 0, 0), gated != 0, h);
    amax = fmaxf(amax, absmax8_f32(h));
  }
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if (lane == 0) s_max[warp] = wmax;
  __syncthreads();
  uint32_t bmax = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) bmax = max(bmax, s_max[w]);
  const float s = __fdiv_rn(static_cast<float>(Q), fmaxf(__uint_as_float(bmax), 1e-5f));
  uint2* qr = reinterpret_cast<uint2*>(Xq + m * K);
  int sum = 0;
  for (int c = t; c < nch; c += kActRowThreads) {
    float h[8];
    relu2_8(__ldg(gr + c), gated ? __ldg(ur + c) : make_uint4(0, 0, 0, 0), gated != 0, h);
    qr[c] = quant8_f32(h, s, sum);
  }
  const int wsum = __reduce_add_sync(0xffffffffu, sum);
  if (lane == 0) s_sum[warp] = wsum;
  __syncthreads();
  if (t == 0) {
    int tot = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) tot += s_sum[w];
    if (s_out) s_out[m] = s;
    if (R_out) R_out[m] = tot;
  }
}

// R[m] = sum_k Xq[m, k] for already-quantised int8 activations.
__global__ void __launch_bounds__(256) bl_act_rowsum_kernel(const int8_t* __restrict__ Xq, int M, int K,
                                                         int* __restrict__ R_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * kActRowsPerBlock + warp;
  if (m >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(Xq + static_cast<size_t>(m) * K);
  int sum = 0;
  for (int c = lane; c < (K >> 4); c += 32) {
    const uint4 v = __ldg(xr + c);
    sum = __dp4a(static_cast<int>(v.x), 0x01010101, sum);
    sum = __dp4a(static_cast<int>(v.y), 0x01010101, sum);
    sum = __dp4a(static_cast<int>(v.z), 0x01010101, sum);
    sum = __dp4a(static_cast<int>(v.w), 0x01010101, sum);
  }
  sum = warp_sum(sum);
  if (lane == 0) R_out[m] = sum;
}

}  // namespace bl
