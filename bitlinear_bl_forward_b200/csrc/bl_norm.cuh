// RMS normalisation of a token right before its absmax quantisation.
//
// "BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs", section "3. Sub-Layer
// Normalization (SubLN)" and the page's pipeline figure: the activations are
// normalised (x_norm = RMSNorm(x)) and then quantised with the per-token
// absmax.  "BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs", table "Best
// Practices for Deploying BitNet a4.8 in Production", row "LayerNorm
// Preservation": the normalisation parameters stay in bf16.
//
// The pages fix no precision; every step here has one exact result:
//   ms  = fp32 round-to-nearest-even of (1/K) sum_k x_k^2, the sum EXACT,
//   r   = __fsqrt_rn(__fadd_rn(ms, eps)),
//   x_n = bf16_rn(__fmul_rn(__fdiv_rn(x, r), w_k))   (w: optional bf16 [K]),
// so the result does not depend on how the sum is split between threads.
//
// Exact sum of squares.  A finite bf16 is sig * 2^(e' - 134) with e' =
// max(e, 1) (e the biased exponent field) and sig < 256, so its square is
// sig^2 * 2^(2e' - 268), a 16-bit integer at bit position P = 2e' + 96 of a
// fixed-point number whose unit is 2^-364.  P runs from 98 to 604 and a sum
// of up to 2^16 squares stays below 2^636: twenty 32-bit limbs.
//   * The block first agrees on E, the largest exponent field of the token.
//     Every thread then adds its squares into a 128-bit register window
//     whose bit 0 sits at position 2E: a square lands at bit
//     96 - 2 (E - e'), exactly, whenever that is >= 0, i.e. for every value
//     within 2^48 of the token's largest.  Warps sum their windows with
//     shuffles (carries kept), and one warp sums the warps' windows: all
//     exact integer additions, so no atomics on this path.
//   * A square further down (a value below 2^-48 of the largest) is added
//     straight into 64-bit limb counters in shared memory at its position.
//     Counters never overflow: such a value is < 2^47 and at most 2^16 of
//     them reach one counter (< 2^63).
//   * Rounding.  Without far squares the window W is the whole sum and
//     ms = RN_f32(W * 2^(2E - 364) / K).  A double estimate
//     q = (double(hi) 2^64 + double(lo)) / K * 2^(2E - 364) is within 2^-51
//     relative of the exact value (three roundings of 2^-53 each plus an
//     exact power-of-two scaling).  If q lies in the normal fp32 range and
//     more than 2^-48 q away from both fp32 midpoints around RN_f32(q), no
//     midpoint separates q from the exact value, so RN_f32(q) is the exact
//     rounding.  Otherwise (a near-tie, far squares, the subnormal or
//     overflow range) the window is folded into the limb counters and one
//     thread takes the exact route: it normalises the counters into 32-bit
//     digits, divides by K digit by digit (a 64-bit multiply-high by
//     ceil(2^64 / K) gives the exact quotient digit because every partial
//     dividend is below 2^48 and K <= 2^16), and rounds on the quotient's
//     bits with the remainder as sticky: normal and subnormal results, ties
//     to even, overflow to infinity.
#pragma once

#include "bl_act.cuh"

namespace bl {

constexpr int kSqLimbs = 20;            // 32-bit limbs of the fixed-point sum
constexpr int kSqWindowShift = 96;      // bit of the anchor's square in the 128-bit window
constexpr int kSqUnitExp = 364;         // unit of the fixed-point sum: 2^-364

// Anchor exponent field of a token from its largest |x| (fp32 bits of a
// bf16 value): the largest exponent field, at least 1.
__device__ __forceinline__ int sq_anchor(uint32_t amax_bits) { return max(static_cast<int>(amax_bits >> 23), 1); }

// One bf16 square (b: the 16-bit pattern) into the thread's window (lo, hi)
// anchored at exponent field E, or into the shared limb counters.  Squares of
// values within 2^16 of the largest land in hi alone (bit 2 (e' - E) + 32 of
// it, < 2^48 each): one 64-bit shift and add.
__device__ __forceinline__ void sq_add1(uint32_t b, int E, unsigned long long& lo, unsigned long long& hi,
                                        unsigned long long* acc) {
  const uint32_t e = (b >> 7) & 0xffu;
  const uint32_t sig = (b & 0x7fu) | (e ? 0x80u : 0u);
  const int ei = e ? static_cast<int>(e) : 1;
  const unsigned long long sq = static_cast<unsigned long long>(sig * sig);
  const int t = 2 * (ei - E) + kSqWindowShift - 64;
  if (t >= 0) {
    hi += sq << t;
    return;
  }
  if (sq == 0ull) return;
  const int sh = t + 64;
  if (sh >= 0) {
    const unsigned long long a_lo = sq << sh;
    const unsigned long long a_hi = sh > 48 ? (sq >> (64 - sh)) : 0ull;
    lo += a_lo;
    hi += a_hi + (lo < a_lo ? 1ull : 0ull);
  } else {
    const int P = 2 * ei + kSqWindowShift;
    atomicAdd(&acc[P >> 5], sq << (P & 31));
  }
}

// Warp sum of the 128-bit windows: every lane holds the total afterwards.
__device__ __forceinline__ void sq_warp_sum(unsigned long long& lo, unsigned long long& hi) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long olo = __shfl_xor_sync(0xffffffffu, lo, o);
    const unsigned long long ohi = __shfl_xor_sync(0xffffffffu, hi, o);
    lo += olo;
    hi += ohi + (lo < olo ? 1ull : 0ull);
  }
}

// Add the window (lo, hi), whose bit 0 sits at position 2E, to the limb
// counters: lane j (0..4) adds 32-bit chunk j.  One warp at a time, every
// lane with the same window; the lanes' counters are distinct.
__device__ __forceinline__ void sq_fold(unsigned long long lo, unsigned long long hi, int E, int lane,
                                        unsigned long long* acc) {
  if (lane < 5) {
    const int B = 2 * E;
    const uint32_t w0 = static_cast<uint32_t>(lo), w1 = static_cast<uint32_t>(lo >> 32);
    const uint32_t w2 = static_cast<uint32_t>(hi), w3 = static_cast<uint32_t>(hi >> 32);
    const uint32_t cur = lane == 0 ? w0 : lane == 1 ? w1 : lane == 2 ? w2 : lane == 3 ? w3 : 0u;
    const uint32_t prev = lane == 0 ? 0u : lane == 1 ? w0 : lane == 2 ? w1 : lane == 3 ? w2 : w3;
    acc[(B >> 5) + lane] += __funnelshift_l(prev, cur, static_cast<uint32_t>(B & 31));
  }
  __syncwarp();
}

// In-place division of the n little-endian 32-bit digits dig by K
// (2 <= K <= 2^16); returns the remainder.  A 64-bit multiply-high by
// ceil(2^64 / K) gives each exact quotient digit: every partial dividend is
// below 2^48, so the estimate's error (< 2^-16) cannot cross an integer.
__device__ __forceinline__ uint32_t digits_div_small(uint32_t* dig, int n, uint32_t K) {
  const unsigned long long inv = ~0ull / K + 1ull;   // ceil(2^64 / K)
  unsigned long long rem = 0;
  for (int i = n - 1; i >= 0; --i) {
    const unsigned long long cur = (rem << 32) | dig[i];
    const unsigned long long q = __umul64hi(cur, inv);
    rem = cur - q * K;
    dig[i] = static_cast<uint32_t>(q);
  }
  return static_cast<uint32_t>(rem);
}

// fp32 round-to-nearest-even of dig * 2^-unit_exp, dig n little-endian
// 32-bit digits (unit_exp >= 150); `below` says whether non-zero bits lie
// below digit 0 (they only break ties).  Normal and subnormal results,
// overflow to infinity.
__device__ float digits_round_f32(const uint32_t* dig, int n, int unit_exp, bool below) {
  int hq = n - 1;
  while (hq > 0 && dig[hq] == 0u) --hq;
  if (dig[hq] == 0u) return 0.f;
  const int Lq = 32 * hq + 31 - __clz(dig[hq]);            // leading bit
  const int kSubLsb = unit_exp - 149;                       // position of 2^-149
  const int lsb = max(Lq - 23, kSubLsb);                    // last kept bit
  if (lsb >= Lq + 2) return 0.f;                            // below half the smallest subnormal
  const int width = Lq - lsb + 1;                           // kept bits, <= 24
  unsigned long long win = dig[lsb >> 5];
  if ((lsb >> 5) + 1 < n) win |= static_cast<unsigned long long>(dig[(lsb >> 5) + 1]) << 32;
  const uint32_t kept0 = static_cast<uint32_t>((win >> (lsb & 31)) & ((1ull << width) - 1ull));
  const int hp = lsb - 1;                                   // the half bit
  const bool half = (dig[hp >> 5] >> (hp & 31)) & 1u;
  bool sticky = below || (dig[hp >> 5] & ((1u << (hp & 31)) - 1u)) != 0u;
  for (int j = 0; j < (hp >> 5) && !sticky; ++j) sticky = dig[j] != 0u;
  const uint32_t kept = kept0 + ((half && (sticky || (kept0 & 1u))) ? 1u : 0u);
  if (lsb > Lq - 23) return __uint_as_float(kept);          // subnormal (rounds up into 2^-126 exactly)
  const int biased = Lq - unit_exp + 127;
  if (biased >= 255) return __uint_as_float(0x7f800000u);
  return __uint_as_float((static_cast<uint32_t>(biased - 1) << 23) + kept);
}

// fp32 round-to-nearest-even of (sum * 2^-364) / K from the limb counters
// (one thread; dig: kSqLimbs words of scratch).
__device__ __noinline__ float sq_mean_f32(const unsigned long long* acc, uint32_t* dig, uint32_t K) {
  unsigned long long carry = 0;
  bool any = false;
  for (int i = 0; i < kSqLimbs; ++i) {
    const unsigned long long t = acc[i] + carry;
    dig[i] = static_cast<uint32_t>(t);
    carry = t >> 32;
    any |= dig[i] != 0u;
  }
  if (!any) return 0.f;
  const uint32_t rem = digits_div_small(dig, kSqLimbs, K);
  return digits_round_f32(dig, kSqLimbs, kSqUnitExp, rem != 0u);
}

// RN_f32(q) for a double q > 0 that lies within 2^-50 (relative) of an exact
// value v: true, with f = RN_f32(v), when q is in the normal fp32 range and
// more than 2^-48 q away from both fp32 midpoints around RN_f32(q) (then no
// midpoint separates q from v); false otherwise (take the exact route).
__device__ __forceinline__ bool f32_round_checked(double q, float& f) {
  if (!(q >= 0x1p-126 && q < 0x1p127)) return false;
  f = __double2float_rn(q);
  const double fd = f;
  const double m_lo = 0.5 * (fd + static_cast<double>(__int_as_float(__float_as_int(f) - 1)));
  const double m_hi = 0.5 * (fd + static_cast<double>(__int_as_float(__float_as_int(f) + 1)));
  const double tol = q * 0x1p-48;
  return q - m_lo > tol && m_hi - q > tol;
}

// The token's mean of squares, by one warp (all 32 lanes) once every
// thread's far squares are in the counters and warp w's window is in
// s_win[2w], s_win[2w + 1] (nw warps, anchored at E).  Returns ms on lane 0.
__device__ __forceinline__ float sq_block_mean(const unsigned long long* s_win, int nw, int E,
                                               unsigned long long* acc, uint32_t* dig, uint32_t K, int lane) {
  unsigned long long lo = lane < nw ? s_win[2 * lane] : 0ull, hi = lane < nw ? s_win[2 * lane + 1] : 0ull;
  sq_warp_sum(lo, hi);
  const bool far = __ballot_sync(0xffffffffu, lane < kSqLimbs && acc[lane] != 0ull) != 0u;
  float ms = 0.f;
  int exact = far ? 1 : 0;
  if (!far && lane == 0 && (lo | hi) != 0ull) {
    const double D = fma(static_cast<double>(hi), 0x1p64, static_cast<double>(lo));
    const double q = (D / static_cast<double>(K)) * __hiloint2double((2 * E - kSqUnitExp + 1023) << 20, 0);
    exact = f32_round_checked(q, ms) ? 0 : 1;
  }
  if (__shfl_sync(0xffffffffu, exact, 0)) {
    sq_fold(lo, hi, E, lane, acc);
    if (lane == 0) ms = sq_mean_f32(acc, dig, K);
  }
  return ms;
}

// ---------------------------------------------------------------------------
// LayerNorm without affine parameters ("BitNet b1.58: The 1-Bit Ternary LLM
// Architecture Guide", BitLinear code listing, forward step 1; the 2B4T
// page's BitLinear module): every step has one exact result,
//   mu  = RN_f32((1/K) sum_k x_k),                      the sum exact,
//   var = RN_f32((1/K) sum_k (x_k - (1/K) sum_j x_j)^2), exact,
//   r   = __fsqrt_rn(__fadd_rn(var, eps)),
//   x_n = bf16_rn(__fdiv_rn(__fsub_rn(x, mu), r)).
//
// Exact sums.  Beside the squares' window above, every thread keeps a signed
// 64-bit window of sum x: a value of exponent field e' (>= 1) and significand
// sig adds +-sig * 2^(e' - E + 38), exact whenever e' >= E - 38 (|window| <
// 2^62 for K <= 2^16).  A value further down goes, like a far square, into
// signed 64-bit limb counters (unit 2^-171, value sig * 2^(e' + 37)).
//   * Fast route (no far value anywhere): with W1 the block's signed window
//     (unit 2^(E - 172)) and S2 its squares' window (unit 2^(2E - 364)),
//         K^2 var = D * 2^(2E - 364),   D = K S2 - W1^2 2^20 >= 0,
//     a 192-bit integer formed exactly.  Double estimates of mu and var are
//     within 2^-50 of the exact values and are rounded when no fp32
//     midpoint is near (f32_round_checked).
//   * Exact route (a far value, a near-tie, a value off the normal range):
//     both windows are folded into the counters and one thread forms |sum x|
//     and sum x^2 as digit strings, divides by K for mu, forms
//     K sum x^2 - (sum x)^2 2^22 (unit 2^-364), divides it by K twice (the
//     two remainders make the sticky bit) and rounds.
// ---------------------------------------------------------------------------

constexpr int kS1Limbs = 11;            // 32-bit limbs of the fixed-point sum of x
constexpr int kS1WindowShift = 38;      // bit of a value of exponent field E in the signed window
constexpr int kS1UnitExp = 171;         // unit of the fixed-point sum: 2^-171
constexpr int kLnDigits = kSqLimbs + 2; // digits of K sum x^2 - (sum x)^2 2^22

// One bf16 value (b: the 16-bit pattern) into the signed window w1 or the
// far counters acc1.
__device__ __forceinline__ void s1_add1(uint32_t b, int E, long long& w1, unsigned long long* acc1) {
  const uint32_t e = (b >> 7) & 0xffu;
  const int sig = static_cast<int>((b & 0x7fu) | (e ? 0x80u : 0u));
  const int ei = e ? static_cast<int>(e) : 1;
  const long long v = (b & 0x8000u) ? -static_cast<long long>(sig) : static_cast<long long>(sig);
  const int sh = ei - E + kS1WindowShift;
  if (sh >= 0) {
    w1 += v * (1ll << sh);
    return;
  }
  if (sig == 0) return;
  const int P = ei + kS1UnitExp - 134;
  atomicAdd(&acc1[P >> 5], static_cast<unsigned long long>(v * (1ll << (P & 31))));
}

// ---------------------------------------------------------------------------
// Per-thread accumulation.  A value x of exponent field e' >= max(E - 16, 1)
// (|x| >= norm_thr(E)) goes into fp64 partial sums p1 = sum x (LayerNorm)
// and p2 = sum x^2, which are exact: such an x is a multiple of
// u1 = 2^(E - 150) below 2^(E - 126), so x is below 2^24 u1 and x^2 a multiple
// of u2 = 2^(2E - 300) below 2^48 u2; up to kNormFlush values keep both sums
// below 2^53 units.  norm_flush then moves them, exactly, into the integer
// windows: p1 / u1 is an integer, times 2^22 in the window's unit
// 2^(E - 172); p2 / u2 is an integer in units of 2^64 of the squares'
// window (its high word).  Values further down (and zeros) take
// s1_add1 / sq_add1.
// ---------------------------------------------------------------------------

constexpr int kNormFlush = 32;          // values between two flushes at most

__device__ __forceinline__ float norm_thr(int E) { return __uint_as_float(static_cast<uint32_t>(max(E - 16, 1)) << 23); }

// Eight bf16 values into the accumulators (p1, w1 and acc1: LayerNorm only).
template <bool LN>
__device__ __forceinline__ void norm_add8(uint4 v, int E, float thr, double& p1, double& p2, long long& w1,
                                          unsigned long long& lo, unsigned long long& hi, unsigned long long* acc1,
                                          unsigned long long* acc2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t xu = (i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16);   // fp32 bits of the value
    if (fabsf(__uint_as_float(xu)) >= thr) {
      // the fp64 value from the fp32 bits of a normal number (exact)
      const double xd = __hiloint2double(static_cast<int>((xu & 0x80000000u) | (((xu & 0x7fffffffu) >> 3) + 0x38000000u)), 0);
      if constexpr (LN) p1 += xd;
      p2 = fma(xd, xd, p2);
    } else {
      if constexpr (LN) s1_add1(xu >> 16, E, w1, acc1);
      sq_add1(xu >> 16, E, lo, hi, acc2);
    }
  }
}

// Move the fp64 partial sums into the integer windows (exact) and reset them.
template <bool LN>
__device__ __forceinline__ void norm_flush(int E, double& p1, double& p2, long long& w1, unsigned long long& hi) {
  if constexpr (LN) {
    const double s1 = __hiloint2double((150 - E + 1023) << 20, 0);        // 1 / u1
    w1 += __double2ll_rn(p1 * s1) * (1ll << 22);
    p1 = 0.0;
  }
  const double s2 = __hiloint2double((300 - 2 * E + 1023) << 20, 0);      // 1 / u2
  hi += __double2ull_rn(p2 * s2);
  p2 = 0.0;
}

// Exact route (one thread): mu and var from the counters.
__device__ __noinline__ void ln_exact(const unsigned long long* acc1, const unsigned long long* acc2, uint32_t K,
                                      float* mu_out, float* var_out) {
  uint32_t a[kS1Limbs], t[kS1Limbs];
  uint32_t d[kLnDigits], c[kLnDigits];
  // sum x: signed counters -> two's complement digits -> sign and magnitude
  long long carry = 0;
  for (int i = 0; i < kS1Limbs; ++i) {
    const long long v = static_cast<long long>(acc1[i]) + carry;
    a[i] = static_cast<uint32_t>(v);
    carry = v >> 32;
  }
  const bool neg = carry < 0;
  if (neg) {
    unsigned long long cy = 1;
    for (int i = 0; i < kS1Limbs; ++i) {
      const unsigned long long v = static_cast<unsigned long long>(~a[i]) + cy;
      a[i] = static_cast<uint32_t>(v);
      cy = v >> 32;
    }
  }
  for (int i = 0; i < kS1Limbs; ++i) t[i] = a[i];
  const uint32_t rem_mu = digits_div_small(t, kS1Limbs, K);
  const float mu = digits_round_f32(t, kS1Limbs, kS1UnitExp, rem_mu != 0u);
  *mu_out = neg ? -mu : mu;
  // K sum x^2 (unit 2^-364)
  unsigned long long cu = 0;
  for (int i = 0; i < kSqLimbs; ++i) {
    const unsigned long long v = acc2[i] + cu;
    d[i] = static_cast<uint32_t>(v);
    cu = v >> 32;
  }
  d[kSqLimbs] = static_cast<uint32_t>(cu);
  d[kSqLimbs + 1] = 0u;
  cu = 0;
  for (int i = 0; i < kLnDigits; ++i) {
    const unsigned long long v = static_cast<unsigned long long>(d[i]) * K + cu;
    d[i] = static_cast<uint32_t>(v);
    cu = v >> 32;
  }
  // (sum x)^2 2^22 (unit 2^-342 -> 2^-364)
  for (int i = 0; i < kLnDigits; ++i) c[i] = 0u;
  for (int i = 0; i < kS1Limbs; ++i) {
    if (a[i] == 0u) continue;
    unsigned long long cy = 0;
    for (int j = 0; j < kS1Limbs && i + j < kLnDigits; ++j) {
      const unsigned long long v = static_cast<unsigned long long>(a[i]) * a[j] + c[i + j] + cy;
      c[i + j] = static_cast<uint32_t>(v);
      cy = v >> 32;
    }
    for (int k = i + kS1Limbs; k < kLnDigits && cy; ++k) {
      const unsigned long long v = static_cast<unsigned long long>(c[k]) + cy;
      c[k] = static_cast<uint32_t>(v);
      cy = v >> 32;
    }
  }
  for (int i = kLnDigits - 1; i > 0; --i) c[i] = (c[i] << 22) | (c[i - 1] >> 10);
  c[0] <<= 22;
  // D = K sum x^2 - (sum x)^2 2^22 >= 0
  long long br = 0;
  for (int i = 0; i < kLnDigits; ++i) {
    const long long v = static_cast<long long>(d[i]) - static_cast<long long>(c[i]) + br;
    d[i] = static_cast<uint32_t>(v);
    br = v >> 32;
  }
  const uint32_t r1 = digits_div_small(d, kLnDigits, K);
  const uint32_t r2 = digits_div_small(d, kLnDigits, K);
  *var_out = digits_round_f32(d, kLnDigits, kSqUnitExp, (r1 | r2) != 0u);
}

// The token's mean and variance, by one warp (all 32 lanes) once every
// thread's far values are in the counters and warp w's windows are in
// s_w1[w], s_win[2w], s_win[2w + 1] (nw warps, anchored at E).  Returns mu
// and var on lane 0.
__device__ __forceinline__ void ln_block_stats(const long long* s_w1, const unsigned long long* s_win, int nw, int E,
                                               unsigned long long* acc1, unsigned long long* acc2, uint32_t K,
                                               int lane, float& mu, float& var) {
  long long w1 = lane < nw ? s_w1[lane] : 0ll;
  unsigned long long lo = lane < nw ? s_win[2 * lane] : 0ull, hi = lane < nw ? s_win[2 * lane + 1] : 0ull;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) w1 += __shfl_xor_sync(0xffffffffu, w1, o);
  sq_warp_sum(lo, hi);
  const bool far = __ballot_sync(0xffffffffu, (lane < kS1Limbs && acc1[lane] != 0ull) ||
                                                   (lane < kSqLimbs && acc2[lane] != 0ull)) != 0u;
  int exact = far ? 1 : 0;
  mu = 0.f;
  var = 0.f;
  if (!far && lane == 0) {
    bool ok = true;
    if (w1 != 0ll) {
      const double q = (fabs(static_cast<double>(w1)) / static_cast<double>(K)) *
                       __hiloint2double((E - kS1WindowShift - 134 + 1023) << 20, 0);
      float f;
      ok = f32_round_checked(q, f);
      mu = w1 < 0 ? -f : f;
    }
    // D = K S2 - W1^2 2^20 over three 64-bit words
    const unsigned long long k = K;
    const unsigned long long a0 = lo * k;
    const unsigned long long m0 = __umul64hi(lo, k);
    const unsigned long long a1 = hi * k + m0;
    const unsigned long long a2 = __umul64hi(hi, k) + (a1 < m0 ? 1ull : 0ull);
    const unsigned long long u = static_cast<unsigned long long>(w1 < 0 ? -w1 : w1);
    const unsigned long long p0 = u * u, p1 = __umul64hi(u, u);
    const unsigned long long b0 = p0 << 20, b1 = (p1 << 20) | (p0 >> 44), b2 = p1 >> 44;
    const unsigned long long d0 = a0 - b0;
    const unsigned long long c0 = a0 < b0 ? 1ull : 0ull;
    const unsigned long long d1 = a1 - b1 - c0;
    const unsigned long long c1 = (a1 < b1 || (a1 == b1 && c0)) ? 1ull : 0ull;
    const unsigned long long d2 = a2 - b2 - c1;
    if ((d0 | d1 | d2) != 0ull && ok) {
      const double D = fma(static_cast<double>(d2), 0x1p128, fma(static_cast<double>(d1), 0x1p64, static_cast<double>(d0)));
      const double q = (D / (static_cast<double>(K) * static_cast<double>(K))) *
                       __hiloint2double((2 * E - kSqUnitExp + 1023) << 20, 0);
      ok = f32_round_checked(q, var);
    }
    exact = ok ? 0 : 1;
  }
  if (__shfl_sync(0xffffffffu, exact, 0)) {
    sq_fold(lo, hi, E, lane, acc2);
    if (lane < 3) {
      // W1 2^(E - 1) (unit 2^-171) as three signed 32-bit pieces
      const int B = E - 1, sh = B & 31;
      const unsigned long long l64 = static_cast<unsigned long long>(w1) << sh;
      const long long top = sh ? (w1 >> (64 - sh)) : (w1 < 0 ? -1ll : 0ll);
      const long long piece = lane == 0 ? static_cast<long long>(static_cast<uint32_t>(l64))
                              : lane == 1 ? static_cast<long long>(static_cast<uint32_t>(l64 >> 32))
                                          : top;
      acc1[(B >> 5) + lane] += static_cast<unsigned long long>(piece);
    }
    __syncwarp();
    if (lane == 0) ln_exact(acc1, acc2, K, &mu, &var);
  }
}

// Normalise 8 bf16 values: bf16_rn(f32(f32(x - mu) / r)).
__device__ __forceinline__ uint4 ln_apply8(uint4 x, float mu, float r) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fdiv_rn(__fsub_rn(bf16_lo(xs[i]), mu), r);
    const float hi = __fdiv_rn(__fsub_rn(bf16_hi(xs[i]), mu), r);
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    o[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Normalise 8 bf16 values: bf16_rn(f32(f32(x / r) * w)), the weight optional.
__device__ __forceinline__ uint4 rms_apply8(uint4 x, uint4 w, bool has_w, float r) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo = __fdiv_rn(bf16_lo(xs[i]), r), hi = __fdiv_rn(bf16_hi(xs[i]), r);
    if (has_w) {
      lo = __fmul_rn(lo, bf16_lo(ws[i]));
      hi = __fmul_rn(hi, bf16_hi(ws[i]));
    }
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    o[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

enum NormKind : int { kNormRms = 0, kNormLayer = 1 };

// RMSNorm (NORM = kNormRms, optional bf16 weight Wn [K]) or LayerNorm
// (kNormLayer, no parameters), then exactly bl_act_quant_row_kernel's
// quantisation of the normalised bf16 row: one CTA per token.  st0: optional
// fp32 [M] mean of squares (RMSNorm) or mean (LayerNorm); st1: optional fp32
// [M] variance (LayerNorm).
constexpr int kNormCache = 4;   // 16-byte chunks a thread keeps in registers (K <= 8192)

template <int NORM>
__global__ void __launch_bounds__(kActRowThreads, 4) bl_act_quant_norm_kernel(
    const uint16_t* __restrict__ X, const uint16_t* __restrict__ Wn, float eps, int K, int Q,
    int8_t* __restrict__ Xq, float* __restrict__ s_out, int* __restrict__ R_out, float* __restrict__ st0,
    float* __restrict__ st1) {
  constexpr int W = kActRowThreads / 32;
  constexpr bool LN = NORM == kNormLayer;
  __shared__ unsigned long long s_sq[kSqLimbs];
  __shared__ unsigned long long s_s1[LN ? kS1Limbs : 1];
  __shared__ unsigned long long s_win[2 * W];
  __shared__ long long s_w1[LN ? W : 1];
  __shared__ uint32_t s_dig[LN ? 1 : kSqLimbs];
  __shared__ float s_r, s_mu;
  __shared__ uint32_t s_max[W];
  __shared__ int s_sum[W];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const size_t m = blockIdx.x;
  if (t < kSqLimbs) s_sq[t] = 0ull;
  if constexpr (LN) {
    if (t < kS1Limbs) s_s1[t] = 0ull;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(X + m * K);
  const uint4* wr = reinterpret_cast<const uint4*>(Wn);
  const bool has_w = !LN && Wn != nullptr;
  const int nch = K >> 3;
  uint4 cache[kNormCache];
  float xmax = 0.f;
#pragma unroll
  for (int i = 0; i < kNormCache; ++i) {
    const int c = t + kActRowThreads * i;
    if (c < nch) {
      cache[i] = __ldg(xr + c);
      xmax = fmaxf(xmax, absmax8_bf16(cache[i]));
    }
  }
  for (int c = t + kActRowThreads * kNormCache; c < nch; c += kActRowThreads)
    xmax = fmaxf(xmax, absmax8_bf16(__ldg(xr + c)));
  const uint32_t wmax_x = __reduce_max_sync(0xffffffffu, __float_as_uint(xmax));
  if (lane == 0) s_max[warp] = wmax_x;
  __syncthreads();   // counters zeroed, per-warp maxima in
  uint32_t xb = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) xb = max(xb, s_max[w]);
  const int E = sq_anchor(xb);
  const float thr = norm_thr(E);
  unsigned long long lo = 0ull, hi = 0ull;
  long long w1 = 0ll;
  double p1 = 0.0, p2 = 0.0;
  static_assert(kNormFlush % 8 == 0 && kNormCache % (kNormFlush / 8) == 0, "flush on chunk boundaries");
#pragma unroll
  for (int i = 0; i < kNormCache; ++i) {
    const int c = t + kActRowThreads * i;
    if (c < nch) norm_add8<LN>(cache[i], E, thr, p1, p2, w1, lo, hi, s_s1, s_sq);
    if ((i + 1) % (kNormFlush / 8) == 0) norm_flush<LN>(E, p1, p2, w1, hi);
  }
  int nf = 0;
  for (int c = t + kActRowThreads * kNormCache; c < nch; c += kActRowThreads) {
    norm_add8<LN>(__ldg(xr + c), E, thr, p1, p2, w1, lo, hi, s_s1, s_sq);
    if (++nf == kNormFlush / 8) {
      norm_flush<LN>(E, p1, p2, w1, hi);
      nf = 0;
    }
  }
  norm_flush<LN>(E, p1, p2, w1, hi);
  sq_warp_sum(lo, hi);
  if constexpr (LN) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w1 += __shfl_xor_sync(0xffffffffu, w1, o);
  }
  if (lane == 0) {
    s_win[2 * warp] = lo;
    s_win[2 * warp + 1] = hi;
    if constexpr (LN) s_w1[warp] = w1;
  }
  __syncthreads();
  if (warp == 0) {
    if constexpr (LN) {
      float mu, var;
      ln_block_stats(s_w1, s_win, W, E, s_s1, s_sq, static_cast<uint32_t>(K), lane, mu, var);
      if (lane == 0) {
        s_mu = mu;
        s_r = __fsqrt_rn(__fadd_rn(var, eps));
        if (st0) st0[m] = mu;
        if (st1) st1[m] = var;
      }
    } else {
      const float ms = sq_block_mean(s_win, W, E, s_sq, s_dig, static_cast<uint32_t>(K), lane);
      if (lane == 0) {
        s_r = __fsqrt_rn(__fadd_rn(ms, eps));
        if (st0) st0[m] = ms;
      }
    }
  }
  __syncthreads();
  const float r = s_r;
  const float mu = LN ? s_mu : 0.f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  auto apply = [&](uint4 x, int c) -> uint4 {
    if constexpr (LN)
      return ln_apply8(x, mu, r);
    else
      return rms_apply8(x, has_w ? __ldg(wr + c) : zero, has_w, r);
  };
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kNormCache; ++i) {
    const int c = t + kActRowThreads * i;
    if (c < nch) {
      cache[i] = apply(cache[i], c);
      amax = fmaxf(amax, absmax8_bf16(cache[i]));
    }
  }
  for (int c = t + kActRowThreads * kNormCache; c < nch; c += kActRowThreads)
    amax = fmaxf(amax, absmax8_bf16(apply(__ldg(xr + c), c)));
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if (lane == 0) s_max[warp] = wmax;
  __syncthreads();
  uint32_t bmax = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) bmax = max(bmax, s_max[w]);
  const float s = __fdiv_rn(static_cast<float>(Q), fmaxf(__uint_as_float(bmax), 1e-5f));
  uint2* qr = reinterpret_cast<uint2*>(Xq + m * K);
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kNormCache; ++i) {
    const int c = t + kActRowThreads * i;
    if (c < nch) qr[c] = quant8_bf16(cache[i], s, sum);
  }
  for (int c = t + kActRowThreads * kNormCache; c < nch; c += kActRowThreads)
    qr[c] = quant8_bf16(apply(__ldg(xr + c), c), s, sum);
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

}  // namespace bl
