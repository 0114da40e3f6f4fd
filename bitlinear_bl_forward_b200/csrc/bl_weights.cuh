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
constexpr int kAbsumWarps = kAbsumThreads / 32;
constexpr int kBins = 256;   // bins 0..253: exponent groups, 255: non-finite count

// Pass 1: per-block exact bins of sum |W|.  out_bins: [gridDim.x][kBins].
__global__ void __launch_bounds__(kAbsumThreads) weight_absum_bins_kernel(const float* __restrict__ W, int64_t n,
                                                                           unsigned long long* __restrict__ out_bins) {
  __shared__ unsigned long long sb[kAbsumWarps][kBins];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kAbsumWarps * kBins; i += blockDim.x) (&sb[0][0])[i] = 0ull;
  __syncthreads();

  const int64_t n4 = n >> 2;   // n is a multiple of 64
  const float4* W4 = reinterpret_cast<const float4*>(W);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // Every lane of the warp runs the same number of iterations so the
  // warp-wide match/reduce below always sees a full warp.
  const int64_t base0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  for (int64_t base = base0; base < n4; base += stride) {
    const int64_t i = base + lane;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n4) v = W4[i];
    const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t u = __float_as_uint(e4[t]) & 0x7fffffffu;
      const uint32_t ex = u >> 23, fr = u & 0x7fffffu;
      uint32_t bin, sig;
      if (ex == 255u) {
        bin = 255u;
        sig = 1u;
      } else if (ex == 0u) {
        bin = 0u;
        sig = fr;
      } else {
        bin = ex - 1u;
        sig = fr | 0x800000u;
      }
      // lanes that share a bin add their significands (< 32 * 2^24) first
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      const unsigned part = __reduce_add_sync(peers, sig);
      if (lane == __ffs(peers) - 1) atomicAdd(&sb[warp][bin], static_cast<unsigned long long>(part));
    }
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
    unsigned long long t = 0;
#pragma unroll
    for (int w = 0; w < kAbsumWarps; ++w) t += sb[w][b];
    out_bins[static_cast<int64_t>(blockIdx.x) * kBins + b] = t;
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

// Pass 2: one block.  Sums the per-block bins and writes gamma.
__global__ void __launch_bounds__(256) weight_gamma_kernel(const unsigned long long* __restrict__ bins, int nblocks,
                                                           uint64_t count, float* __restrict__ gamma) {
  __shared__ unsigned long long tot[kBins];
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
    unsigned long long t = 0;
    for (int g = 0; g < nblocks; ++g) t += bins[static_cast<int64_t>(g) * kBins + b];
    tot[b] = t;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (tot[255] != 0ull) {   // a non-finite weight
    *gamma = __int_as_float(0x7fc00000);
    return;
  }
  // S = sum_b tot[b] * 2^b, in units of 2^-149; tot[b] < 2^64, b <= 253
  constexpr int kLimbs = 12;
  uint32_t S[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) S[i] = 0;
  for (int b = 0; b < 254; ++b) {
    const unsigned long long v = tot[b];
    if (!v) continue;
    const int li = b >> 5, sh = b & 31;
    // v << sh spans up to three limbs
    uint32_t part[3];
    part[0] = static_cast<uint32_t>(v << sh);
    part[1] = static_cast<uint32_t>(sh ? (v >> (32 - sh)) : (v >> 32));
    part[2] = static_cast<uint32_t>(sh ? (v >> (64 - sh)) : 0ull);
    uint64_t carry = 0;
    for (int k = li; k < kLimbs; ++k) {
      const uint64_t add = (k - li < 3) ? part[k - li] : 0u;
      const uint64_t s = static_cast<uint64_t>(S[k]) + add + carry;
      S[k] = static_cast<uint32_t>(s);
      carry = s >> 32;
      if (k - li >= 2 && carry == 0) break;
    }
  }
  const float mean = round_ratio_to_f32(S, kLimbs, count);
  *gamma = fmaxf(mean, 1e-5f);
}

// Pass 3: ternary codes and packing, one thread per 32-bit output word.
__global__ void __launch_bounds__(256) weight_pack_kernel(const float* __restrict__ W, int64_t nwords,
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
__global__ void __launch_bounds__(256) weight_unpack_kernel(const uint32_t* __restrict__ Wp, int64_t nwords,
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

}  // namespace bl
