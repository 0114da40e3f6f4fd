// One-token BitLinear forward (decode), built for back-to-back launches.
//
// What it computes is the one-token case of the BitLinear forward of "BitNet
// b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear" (absmean ternary weights, eq. (1);
// per-token absmax int8 activations, eq. (2); integer matmul and one rescale,
// eq. (3)): y = f32(f32(sum_k c*q) * f32(gamma/s)), the sum taken exactly in
// integers (each ternary weight adds, subtracts or skips an activation: the
// same page, section "Why 1.58 Bits? The Power of Zero").
//
// The shape of the work: every weight byte is read once, the token is 5-16 KB,
// and a whole decode layer is a few MB, i.e. well under a microsecond of HBM
// time.  So the kernel is organised around hiding latency between launches:
//
//   * a launch has exactly one CTA per SM (rows split evenly, so no SM holds
//     two CTAs of one launch and none waits with no work), a CTA takes a
//     little under half an SM (104 KB of shared memory, <= 112 registers a
//     thread at 8 consumer warps, <= 60 at 16), so the CTAs of the next
//     launch on the stream (programmatic dependent launch, triggered at the
//     start of this one) become resident beside this launch's CTAs;
//   * the weights are constant parameters, not produced by the preceding
//     kernel: a producer warp fetches this CTA's first ring stages (cp.async.bulk
//     into shared memory) BEFORE the dependency wait, i.e. while the previous
//     launch is still running, and only the consumers wait for the token;
//   * consumers: quantise the token (absmax per token, Q/max(a, eps), round to
//     nearest even, clamp; optionally after squared ReLU or RMSNorm, formed
//     in the same prologue), keep it, then for each weight row:
//     lane l takes the 32-bit words l, l+32, ... (16 weights each; balanced for
//     every K that is a multiple of 64), four masked unsigned-by-signed dp4a
//     per word (slice j of a word holds 4^j * (c+1) in each byte), exact fold
//     acc0 + acc1/4 + acc2/16 + acc3/64, one warp redux per row, offset
//     correction sum_k (c+1) q - sum_k q, fp32 rescale, store.
#pragma once

#include "bl_act.cuh"
#include "bl_gemv.cuh"
#include "bl_norm.cuh"

namespace bl {

constexpr int kG3Stages = 3;
constexpr int kG3StageBytes = 32768;
constexpr int kG3MaxK = 8192;
// dynamic shared memory: [3 x 32 KB weight ring][token codes, 8 KB]
constexpr int kG3SmemBytes = kG3Stages * kG3StageBytes + kG3MaxK;

// What the token prologue forms before the quantisation: nothing (bf16
// activations or int8 codes), the squared-ReLU input, or the RMS-normalised
// token.  A template parameter so that the plain path carries no code for
// the others.
enum G3Pre : int { kG3Plain = 0, kG3Relu2 = 1, kG3Rms = 2 };

template <int WPL, int CW>
struct G3Cfg {
  static constexpr int kThreads = (CW + 1) * 32;   // CW consumer warps + 1 producer warp
  // the token codes stay in registers for small K; for large K each lane
  // reads them from shared memory next to the weight word (one extra load a
  // word shared by two rows, but registers for 16 warps)
  static constexpr bool kActSmem = WPL > 6;
};

// RT rows of one stage for one warp: partial dot products of lane's words,
// folded slices, warp sum, offset correction, rescale, store.
template <int RT, int WPL, bool ACT_SMEM>
__device__ __forceinline__ void g3_rows(const uint8_t* sbase, int rr, int rows, int row_bytes, int words, int lane,
                                        const uint32_t (&act)[ACT_SMEM ? 1 : WPL][4], const uint8_t* s_act,
                                        int row0, int R, float f, void* __restrict__ Y, int out_mode,
                                        const float* __restrict__ bias) {
  const uint32_t* p[RT];
  bool live[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    p[r] = reinterpret_cast<const uint32_t*>(sbase + (rr + r) * row_bytes);
    live[r] = (r == 0) || (rr + r < rows);
  }
  int acc[RT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[r][j] = 0;
#pragma unroll(ACT_SMEM ? 2 : WPL)
  for (int i = 0; i < WPL; ++i) {
    const int wi = lane + 32 * i;
    const bool in = i < WPL - 1 || wi < words;
    uint32_t w[RT];
#pragma unroll
    for (int r = 0; r < RT; ++r) w[r] = (live[r] && in) ? p[r][wi] : 0u;
    uint32_t a[4];
    if constexpr (ACT_SMEM) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (in) v = *reinterpret_cast<const uint4*>(&s_act[16 * wi]);
      a[0] = v.x;
      a[1] = v.y;
      a[2] = v.z;
      a[3] = v.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) a[j] = act[i][j];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int r = 0; r < RT; ++r) acc[r][j] = dp4a_us(w[r] & (0x03030303u << (2 * j)), a[j], acc[r][j]);
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const int part = acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6);
    const int tot = __reduce_add_sync(0xffffffffu, part);
    const int n = row0 + rr + r;
    if (lane == r && rr + r < rows) {
      const int v = tot - R;
      if (out_mode == kOutI32) {
        static_cast<int*>(Y)[n] = v;
      } else {
        float y = __fmul_rn(__int2float_rn(v), f);
        if (bias) y = __fadd_rn(y, __ldg(bias + n));
        if (out_mode == kOutF32)
          static_cast<float*>(Y)[n] = y;
        else
          static_cast<__nv_bfloat16*>(Y)[n] = __float2bfloat16_rn(y);
      }
    }
  }
}

template <int WPL, int CW, int PRE>
__global__ void __launch_bounds__(G3Cfg<WPL, CW>::kThreads, 2)
    gemv3_kernel(const __grid_constant__ G2Table tab, int in_mode, int Q, int out_mode, unsigned long long limit_ns) {
  constexpr bool ACT_SMEM = G3Cfg<WPL, CW>::kActSmem;
  constexpr bool RELU2 = PRE == kG3Relu2;
  constexpr bool RMS = PRE == kG3Rms;
  int pi = 0;
  while (pi + 1 < tab.count && static_cast<int>(blockIdx.x) >= tab.p[pi + 1].cta_begin) ++pi;
  const void* __restrict__ X = tab.p[pi].X;
  const void* __restrict__ Up = tab.p[pi].U;
  const uint8_t* __restrict__ Wp = tab.p[pi].Wp;
  const float* __restrict__ gamma_p = tab.p[pi].gamma;
  void* __restrict__ Y = tab.p[pi].Y;
  const float* __restrict__ bias = tab.p[pi].bias;
  const int K = tab.p[pi].K, N = tab.p[pi].N, ctas = tab.p[pi].ctas;
  const int cta = static_cast<int>(blockIdx.x) - tab.p[pi].cta_begin;

  extern __shared__ __align__(128) uint8_t g3_smem[];
  uint8_t* const s_act = g3_smem + kG3Stages * kG3StageBytes;
  static_assert(CW % 4 == 0, "partials are read four at a time");
  __shared__ __align__(16) uint32_t s_red_f[CW];
  __shared__ __align__(16) int s_red_i[CW];
  __shared__ __align__(8) uint64_t full[kG3Stages], empty[kG3Stages];
  __shared__ int abort_flag;
  __shared__ unsigned long long s_sq[RMS ? kSqLimbs : 1];
  __shared__ unsigned long long s_win[RMS ? 2 * CW : 1];
  __shared__ uint32_t s_dig[RMS ? kSqLimbs : 1];
  __shared__ float s_rms;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = K >> 4;
  const int row_bytes = K >> 2;
  const int r0 = static_cast<int>(static_cast<int64_t>(cta) * N / ctas);
  const int r1 = static_cast<int>(static_cast<int64_t>(cta + 1) * N / ctas);
  // rows a ring stage holds; a multiple of two rows per warp when it fits
  int stage_rows = kG3StageBytes / row_bytes;
  if (stage_rows >= 2 * CW) stage_rows -= stage_rows % (2 * CW);
  const int nst = (r1 > r0) ? (r1 - r0 + stage_rows - 1) / stage_rows : 0;
  volatile int* abort_v = &abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kG3Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (RMS) {
    if (threadIdx.x < kSqLimbs) s_sq[threadIdx.x] = 0ull;
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == CW) {
    // ---------------- producer (never waits on the preceding kernel) ----------------
    if (lane == 0) {
      const uint8_t* base = Wp + static_cast<size_t>(r0) * row_bytes;
      const int pre = min(nst, kG3Stages);
      for (int st = 0; st < pre; ++st) {
        const int rows = min(stage_rows, r1 - (r0 + st * stage_rows));
        const uint32_t bytes = static_cast<uint32_t>(rows * row_bytes);
        mbar_arrive_expect_tx(&full[st], bytes);
        bulk_load(g3_smem + st * kG3StageBytes, base + static_cast<size_t>(st) * stage_rows * row_bytes, bytes,
                  &full[st]);
      }
      if (nst > pre) {   // the rest of this CTA's rows: towards L2 now
        const size_t off0 = static_cast<size_t>(pre) * stage_rows * row_bytes;
        const size_t bytes = static_cast<size_t>(r1 - r0) * row_bytes;
        for (size_t off = off0; off < bytes; off += kPrefetchChunk)
          bulk_prefetch_l2(base + off, static_cast<uint32_t>(min(static_cast<size_t>(kPrefetchChunk), bytes - off)));
      }
      int issued = pre;
      for (int st = pre; st < nst; ++st) {
        const int s = st % kG3Stages;
        if (!mbar_wait(&empty[s], ((st / kG3Stages) & 1) ^ 1u, abort_v, limit_ns, 21)) break;
        const int rows = min(stage_rows, r1 - (r0 + st * stage_rows));
        const uint32_t bytes = static_cast<uint32_t>(rows * row_bytes);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(g3_smem + s * kG3StageBytes, base + static_cast<size_t>(st) * stage_rows * row_bytes, bytes,
                  &full[s]);
        issued = st + 1;
      }
      // no copy may be in flight when the CTA exits
      for (int s = 0; s < kG3Stages && s < issued; ++s) {
        const int last = s + kG3Stages * ((issued - 1 - s) / kG3Stages);
        mbar_wait(&full[s], (last / kG3Stages) & 1, nullptr, limit_ns, 22);
      }
    }
    return;
  }

  // ---------------- consumers: the token (written by the preceding kernel) ----------------
  constexpr int CT = CW * 32;
  constexpr int U = (kG3MaxK / 8 + CT - 1) / CT;
  // the norm's weight is a parameter like Wp: fetched before the wait
  uint4 nw[RMS ? U : 1];
  const bool has_nw = RMS && Up != nullptr;
  if constexpr (RMS) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + CT * u;
      nw[u] = (has_nw && c < (K >> 3)) ? __ldg(static_cast<const uint4*>(Up) + c) : make_uint4(0, 0, 0, 0);
    }
  }
  pdl_wait();
  const bool x_is_i8 = in_mode == kInI8;
  constexpr bool relu2 = RELU2;
  const bool gated = RELU2 && in_mode == kInRelu2Gated;
  const int nch = x_is_i8 ? (K >> 4) : (K >> 3);
  uint4 xv[U], uv[RELU2 ? U : 1];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = threadIdx.x + CT * u;
    xv[u] = (c < nch) ? __ldg(static_cast<const uint4*>(X) + c) : make_uint4(0, 0, 0, 0);
    if constexpr (RELU2) uv[u] = (gated && c < nch) ? __ldg(static_cast<const uint4*>(Up) + c) : make_uint4(0, 0, 0, 0);
  }
  if constexpr (RMS) {
    // exact mean of squares (register windows anchored at the token's
    // largest exponent, far squares in shared limb counters), then
    // x_n = bf16(x / sqrt(ms + eps) * w) in place of the token
    float xmax = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (threadIdx.x + CT * u < nch) xmax = fmaxf(xmax, absmax8_bf16(xv[u]));
    const uint32_t wmax_x = __reduce_max_sync(0xffffffffu, __float_as_uint(xmax));
    if (lane == 0) s_red_f[warp] = wmax_x;
    named_bar_sync(1, CT);
    uint32_t xb = 0;
#pragma unroll
    for (int w = 0; w < CW; w += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(&s_red_f[w]);
      xb = max(xb, max(max(v.x, v.y), max(v.z, v.w)));
    }
    const int E = sq_anchor(xb);
    unsigned long long lo = 0ull, hi = 0ull;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (threadIdx.x + CT * u < nch) sq_add8(xv[u], E, lo, hi, s_sq);
    sq_warp_sum(lo, hi);
    if (lane == 0) {
      s_win[2 * warp] = lo;
      s_win[2 * warp + 1] = hi;
    }
    named_bar_sync(1, CT);
    if (warp == 0) {
      const float ms = sq_block_mean(s_win, CW, E, s_sq, s_dig, static_cast<uint32_t>(K), lane);
      if (lane == 0) s_rms = __fsqrt_rn(__fadd_rn(ms, tab.p[pi].eps));
    }
    named_bar_sync(1, CT);
    const float r = s_rms;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (threadIdx.x + CT * u < nch) xv[u] = rms_apply8(xv[u], nw[u], has_nw, r);
  }
  const float gamma = (out_mode == kOutI32) ? 1.f : __ldg(gamma_p);
  int rsum = 0;
  float sc = 1.f;
  if (!x_is_i8) {
    float amax = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if constexpr (RELU2) {
        float h[8];
        relu2_8(xv[u], uv[u], gated, h);
        amax = fmaxf(amax, absmax8_f32(h));
      } else {
        amax = fmaxf(amax, absmax8_bf16(xv[u]));
      }
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0) s_red_f[warp] = wmax;
    named_bar_sync(1, CT);
    uint32_t bmax = 0;
#pragma unroll
    for (int w = 0; w < CW; w += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(&s_red_f[w]);
      bmax = max(bmax, max(max(v.x, v.y), max(v.z, v.w)));
    }
    sc = __fdiv_rn(static_cast<float>(Q), fmaxf(__uint_as_float(bmax), 1e-5f));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + CT * u;
      if (c < nch) {
        if constexpr (RELU2) {
          float h[8];
          relu2_8(xv[u], uv[u], gated, h);
          *reinterpret_cast<uint2*>(&s_act[8 * c]) = quant8_f32(h, sc, Q, rsum);
        } else {
          *reinterpret_cast<uint2*>(&s_act[8 * c]) = quant8_bf16(xv[u], sc, Q, rsum);
        }
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + CT * u;
      if (c < nch) {
        const uint4 v = xv[u];
        rsum = __dp4a(static_cast<int>(v.x), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.y), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.z), 0x01010101, rsum);
        rsum = __dp4a(static_cast<int>(v.w), 0x01010101, rsum);
        *reinterpret_cast<uint4*>(&s_act[16 * c]) = v;
      }
    }
  }
  {
    const int ws = __reduce_add_sync(0xffffffffu, rsum);
    if (lane == 0) s_red_i[warp] = ws;
  }
  const float f = (x_is_i8 || out_mode == kOutI32) ? 0.f : __fdiv_rn(gamma, sc);
  named_bar_sync(1, CT);
  int R = 0;
#pragma unroll
  for (int w = 0; w < CW; w += 4) {
    const int4 v = *reinterpret_cast<const int4*>(&s_red_i[w]);
    R += (v.x + v.y) + (v.z + v.w);
  }

  // the 16 activation codes of word (lane + 32 i), four per register (slice j)
  uint32_t act[ACT_SMEM ? 1 : WPL][4];
  if constexpr (!ACT_SMEM) {
#pragma unroll
    for (int i = 0; i < WPL; ++i) {
      const int wi = lane + 32 * i;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (i < WPL - 1 || wi < words) v = *reinterpret_cast<const uint4*>(&s_act[16 * wi]);
      act[i][0] = v.x;
      act[i][1] = v.y;
      act[i][2] = v.z;
      act[i][3] = v.w;
    }
  }

  // ---------------- consumers: weight rows from the ring ----------------
  for (int st = 0; st < nst; ++st) {
    const int s = st % kG3Stages;
    const bool ok = mbar_wait(&full[s], (st / kG3Stages) & 1, abort_v, limit_ns, 23);
    if (!__all_sync(0xffffffffu, ok)) break;
    const int row0 = r0 + st * stage_rows;
    const int rows = min(stage_rows, r1 - row0);
    const uint8_t* sbase = g3_smem + s * kG3StageBytes;
    if (rows > CW) {   // some warp has two rows: take them together
      for (int rr = warp * 2; rr < rows; rr += CW * 2)
        g3_rows<2, WPL, ACT_SMEM>(sbase, rr, rows, row_bytes, words, lane, act, s_act, row0, R, f, Y, out_mode, bias);
    } else if (warp < rows) {
      g3_rows<1, WPL, ACT_SMEM>(sbase, warp, rows, row_bytes, words, lane, act, s_act, row0, R, f, Y, out_mode, bias);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace bl
