// Weight quantisation: absmean scale, ternary codes and 2-bit packing.
//
// "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear", eq. (1) (weight quantisation,
// absmean scaling): gamma = (1/nm) * sum |W_ij| and
// W~ = Round(Clip(W / (gamma + eps), -1, 1)).  The library reads eps as a
// floor, gamma = max(mean|W|, 1e-5), as the code listings on the same pages do
// (clamp(min=1e-5)).
//
// gamma is made independent of the reduction order: every |w| is an integer
// multiple of 2^-149, the kernels add the significands exactly into 64-bit
// bins keyed by exponent, and one thread turns the bins into a multi-word
// integer and divides it by N*K with a single round-to-nearest-even to fp32.
//
// 2-bit storage (this library's format; the pages fix only "2 bits per
// weight"):  row n starts at byte n*K/4 and is a sequence of little-endian
// 32-bit words; word g holds weights k = 16g..16g+15; weight k = 16g + 4j + b
// sits in bits [8b + 2j, 8b + 2j + 2) and stores u = code + 1 (0 -> -1,
// 1 -> 0, 2 -> +1).  With this placement (word >> 2j) & 0x03030303 yields the
// four codes of k = 16g + 4j .. 16g + 4j + 3 as four bytes, i.e. one int8x4
// lane-aligned with four consecutive activation bytes.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kAbsumThreads = 256;
constexpr int kAbsumChunks = 9;     // |w| * 2^149 < 2^277: nine 32-bit positions (+ carry)
constexpr int kAbsumTotals = 16;    // global accumulators: limbs 0..9, [15] = non-finite count

// Pass 1: the exact sum of |W| in units of 2^-149, as 32-bit limbs.
// Every |w| is sig * 2^b * 2^-149 with sig < 2^24 and b = 0..253; a thread
// adds the two 32-bit pieces of sig << (b % 32) to its own positional
// accumulators b / 32 and b / 32 + 1 (private columns of a shared-memory
// array: conflict-free whatever the exponents), the block sums them, carries
// them into 32-bit limbs and adds those to total[0..9].  All additions are
// exact integer additions (bounds: a thread sees < 2^23 elements, a block
// < 2^31, so no accumulator can overflow), hence no dependence on the order.
// total must be zero before the launch.
__global__ void __launch_bounds__(kAbsumThreads) bl_weight_absum_kernel(const float* __restrict__ W, int64_t n,
                                                                           unsigned long long* __restrict__ total) {
  __shared__ unsigned long long acc[kAbsumChunks + 1][kAbsumThreads];
  __shared__ unsigned long long red[kAbsumChunks + 1];
  const int tid = threadIdx.x;
#pragma unroll
  for (int c = 0; c <= kAbsumChunks; ++c) acc[c][tid] = 0ull;
  if (tid <= kAbsumChunks) red[tid] = 0ull;
  unsigned int nonfinite = 0;
  const int64_t n4 = n >> 2;   // n is a multiple of 64
  const float4* W4 = reinterpret_cast<const float4*>(W);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid; i < n4; i += stride) {
    const float4 v = __ldg(W4 + i);
    const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t u = __float_as_uint(e4[e]) & 0x7fffffffu;
      const uint32_t ex = u >> 23, fr = u & 0x7fffffu;
      if (ex == 255u) {
        ++nonfinite;
        continue;
      }
      // normal: (fr + 2^23) * 2^(ex - 150) = sig * 2^(ex - 1) * 2^-149; subnormal: fr * 2^-149
      const uint32_t b = ex ? ex - 1u : 0u;
      const uint32_t sig = ex ? (fr | 0x800000u) : fr;
      const unsigned long long piece = static_cast<unsigned long long>(sig) << (b & 31u);
      const uint32_t c = b >> 5;
      acc[c][tid] += piece & 0xffffffffull;
      acc[c + 1][tid] += piece >> 32;
    }
  }
  __syncthreads();
  // column sums: warp w adds up chunk c = w, w + 8 over the 256 threads
  const int warp = tid >> 5, lane = tid & 31;
  for (int c = warp; c <= kAbsumChunks; c += kAbsumThreads / 32) {
    unsigned long long t = 0;
    for (int k = lane; k < kAbsumThreads; k += 32) t += acc[c][k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) red[c] = t;
  }
  const unsigned int nf = __reduce_add_sync(0xffffffffu, nonfinite);
  if (lane == 0 && nf) atomicAdd(&total[kAbsumTotals - 1], static_cast<unsigned long long>(nf));
  __syncthreads();
  if (tid == 0) {
    unsigned long long carry = 0;
    for (int c = 0; c <= kAbsumChunks; ++c) {
      const unsigned long long t = red[c] + carry;   // red[c] < 2^63
      const unsigned long long limb = t & 0xffffffffull;
      carry = t >> 32;
      if (limb) atomicAdd(&total[c], limb);
    }
    if (carry) atomicAdd(&total[kAbsumChunks + 1 < kAbsumTotals - 1 ? kAbsumChunks + 1 : 0], carry);
  }
}

// Round (S * 2^-149) / D to fp32, nearest-even.  S is a little-endian array of
// 32-bit limbs.  Results below the normal range return 0 (the caller floors
// gamma at 1e-5, far above it).
__device__ float round_ratio_to_f32(const uint32_t* S, int nlimbs, uint64_t D) {
  int ls = 0;   // bit length of S
  for (int i = nlimbs - 1; i >= 0; --i)
    if (S[i]) {
      ls = 32 * i + (32 - __clz(S[i]));
      break;
    }
  if (ls == 0) return 0.f;
  const int ld = 64 - __clzll(static_cast<long long>(D));
  // numerator S * 2^t with t chosen so the quotient has at least 26 bits
  int t = 26 + ld - ls;
  if (t < 0) t = 0;
  const int nbits = ls + t;
  uint64_t r = 0;
  int top = -1;          // index of the leading quotient bit
  uint32_t mant = 0;     // leading 24 quotient bits
  int got = 0;           // quotient bits collected into mant (max 24)
  uint32_t round_bit = 0, sticky = 0;
  for (int i = nbits - 1; i >= 0; --i) {
    const int si = i - t;
    const uint32_t bit = (si >= 0) ? ((S[si >> 5] >> (si & 31)) & 1u) : 0u;
    r = (r << 1) | bit;
    uint32_t q = 0;
    if (r >= D) {
      r -= D;
      q = 1;
    }
    if (top < 0) {
      if (q) {
        top = i;
        mant = 1;
        got = 1;
      }
    } else if (got < 24) {
      mant = (mant << 1) | q;
      ++got;
    } else if (got == 24) {
      round_bit = q;
      ++got;
    } else {
      sticky |= q;
    }
  }
  if (r != 0) sticky = 1;
  // value = (quotient) * 2^(-149 - t); leading bit at index `top`
  int E = top - 149 - t;
  if (round_bit && (sticky || (mant & 1u))) {
    ++mant;
    if (mant == (1u << 24)) {
      mant >>= 1;
      ++E;
    }
  }
  if (E < -126) return 0.f;
  if (E > 127) return __int_as_float(0x7f800000);
  return __uint_as_float((static_cast<uint32_t>(E + 127) << 23) | (mant & 0x7fffffu));
}

// Pass 2: one thread.  Turns the limb totals into gamma.
__global__ void __launch_bounds__(32) bl_weight_gamma_kernel(const unsigned long long* __restrict__ total, uint64_t count,
                                                          float* __restrict__ gamma) {
  if (threadIdx.x != 0) return;
  if (total[kAbsumTotals - 1] != 0ull) {   // a non-finite weight
    *gamma = __int_as_float(0x7fc00000);
    return;
  }
  // S = sum_c total[c] * 2^(32 c), in units of 2^-149; total[c] < 2^42
  constexpr int kLimbs = 14;
  uint32_t S[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) S[i] = 0;
  unsigned long long carry = 0;
  for (int c = 0; c < kLimbs; ++c) {
    const unsigned long long t = (c < kAbsumTotals - 1 ? total[c] : 0ull) + carry;
    S[c] = static_cast<uint32_t>(t);
    carry = t >> 32;
  }
  const float mean = round_ratio_to_f32(S, kLimbs, count);
  *gamma = fmaxf(mean, 1e-5f);
}

// Pass 3: ternary codes and packing, one thread per 32-bit output word.
__global__ void __launch_bounds__(256) bl_weight_pack_kernel(const float* __restrict__ W, int64_t nwords,
                                                          const float* __restrict__ gamma_p,
                                                          uint32_t* __restrict__ Wp) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nwords) return;
  const float gamma = *gamma_p;
  const float4* src = reinterpret_cast<const float4*>(W) + g * 4;   // 16 consecutive weights (same row)
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 v = src[j];   // k = 16g' + 4j .. +3 -> b = 0..3
    const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int c = __float2int_rn(__fdiv_rn(e4[b], gamma));
      c = c < -1 ? -1 : (c > 1 ? 1 : c);
      word |= static_cast<uint32_t>(c + 1) << (8 * b + 2 * j);
    }
  }
  Wp[g] = word;
}

// Packed words -> int8 codes, one thread per word (16 codes, one uint4 out).
__global__ void __launch_bounds__(256) bl_weight_unpack_kernel(const uint32_t* __restrict__ Wp, int64_t nwords,
                                                            int8_t* __restrict__ codes) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nwords) return;
  const uint32_t w = Wp[g];
  uint32_t out[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // bytes b = 0..3 of this output word are codes k = 16g + 4j + b
    const uint32_t u = (w >> (2 * j)) & 0x03030303u;
    // subtract 1 from each byte: u in {0,1,2} per byte; 0 - 1 must become 0xff
    out[j] = ((u | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
  }
  reinterpret_cast<uint4*>(codes)[g] = make_uint4(out[0], out[1], out[2], out[3]);
}

// ---------------------------------------------------------------------------
// Base-3 storage: five ternary weights per byte (3^5 = 243 states fit in a
// byte: "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section
// "Why 1.58 Bits? The Power of Zero", log2(3) ~ 1.58 bits a weight).  Layout
// (this library's): a row is base3 words padded to a multiple of four (16
// bytes); byte b of little-endian word g holds the digits d_L = code + 1 of
// weights k = 20g + 4L + b (L = 0..4, digits past the row end are 1) as
// ceil(256 * v / 243), v = sum_L d_L 3^(4-L).  Level L of the four bytes of a
// word is then four consecutive weights, and a decoder gets the levels in
// order by tripling each byte (digit = (3x) >> 8, next x = 3x mod 256).
// ---------------------------------------------------------------------------

__host__ __device__ constexpr int base3_row_words(int K) { return ((K + 19) / 20 + 3) / 4 * 4; }

// One thread per output word: 20 weights -> four bytes.
__global__ void __launch_bounds__(256) bl_weight_pack3_kernel(const float* __restrict__ W, int N, int K,
                                                           const float* __restrict__ gamma_p,
                                                           uint32_t* __restrict__ Wp3) {
  const int rw = base3_row_words(K);
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(N) * rw) return;
  const int n = static_cast<int>(idx / rw), g = static_cast<int>(idx % rw);
  const float gamma = *gamma_p;
  const float* row = W + static_cast<size_t>(n) * K;
  uint32_t word = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    int v = 0;
#pragma unroll
    for (int L = 0; L < 5; ++L) {
      const int k = 20 * g + 4 * L + b;
      int d = 1;   // padding: code 0
      if (k < K) {
        int c = __float2int_rn(__fdiv_rn(__ldg(row + k), gamma));
        c = c < -1 ? -1 : (c > 1 ? 1 : c);
        d = c + 1;
      }
      v = 3 * v + d;
    }
    word |= static_cast<uint32_t>((256 * v + 242) / 243) << (8 * b);
  }
  Wp3[idx] = word;
}

// Base-3 words -> int8 codes [N, K], one thread per word (up to 20 codes).
__global__ void __launch_bounds__(256) bl_weight_unpack3_kernel(const uint32_t* __restrict__ Wp3, int N, int K,
                                                             int8_t* __restrict__ codes) {
  const int rw = base3_row_words(K);
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(N) * rw) return;
  const int n = static_cast<int>(idx / rw), g = static_cast<int>(idx % rw);
  const uint32_t w = Wp3[idx];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t x = (w >> (8 * b)) & 0xffu;
#pragma unroll
    for (int L = 0; L < 5; ++L) {
      const uint32_t t = 3u * x;
      const int k = 20 * g + 4 * L + b;
      if (k < K) codes[static_cast<size_t>(n) * K + k] = static_cast<int8_t>(static_cast<int>(t >> 8) - 1);
      x = t & 0xffu;
    }
  }
}

}  // namespace bl
