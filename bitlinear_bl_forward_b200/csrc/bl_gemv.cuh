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
    bl_decode_long_kernel(const void* __restrict__ X, int x_is_i8, int M, int K, int N, const uint4* __restrict__ Wp,
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
        const uint2 q = quant8_bf16(__ldg(xr + c), s, rsum);
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


// ---------------------------------------------------------------------------
// Decode fast path: MT in {1, 2} tokens, K <= 8192 (CPL = ceil(K/64/32) <= 4).
//
//   1. each CTA owns a contiguous range of output rows, i.e. one contiguous
//      byte range of packed weights; one thread asks the TMA unit to stream
//      that range into L2 (cp.async.bulk.prefetch.L2).  Then the programmatic
//      dependent-launch handshake: nothing before griddepcontrol.wait reads
//      or writes memory, so an early start is safe whatever precedes it;
//   2. the CTA quantises the token(s) once (two block barriers) into shared
//      memory, XOR-swizzled so that the lanes' 64-byte-strided reads hit
//      distinct banks; lane l then keeps the int8 activations of its
//      64-weight chunks l, l+32, ... in registers for every row it visits;
//   3. each warp walks RT-row tiles of the CTA's range and double-buffers the
//      packed weights of two tiles in registers;
//   4. unpacking without shifts: for the 2-bit slice j of a word,
//      (w & (0x03030303 << 2j)) holds 4^j * u per byte, so an unsigned x
//      signed dp4a gives 4^j * sum u*q; each slice has its own accumulator
//      and the exact total is acc0 + (acc1 >> 2) + (acc2 >> 4) + (acc3 >> 6)
//      (every acc_j is a multiple of 4^j; |acc_3| <= 64*2*127*K/4 < 2^31);
//   5. warp-shuffle reduction, offset correction, rescale, store.
// ---------------------------------------------------------------------------
constexpr uint32_t kPrefetchChunk = 1u << 16;

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <int CPL, int RT>
__device__ __forceinline__ void gemv1_load(uint4 (&w)[RT][CPL], const uint4* __restrict__ Wp, int tile, int tend,
                                           int N, int KV, int lane) {
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int n = tile * RT + r, c = lane + 32 * i;
      w[r][i] = (tile < tend && n < N && c < KV) ? ldg_pinned_v4(Wp + static_cast<size_t>(n) * KV + c)
                                                 : make_uint4(0, 0, 0, 0);
    }
}

// Partial dot products of one RT-row tile for this lane: one accumulator per
// token and 2-bit slice j (each a multiple of 4^j), folded into one partial.
template <int MT, int CPL, int RT>
__device__ __forceinline__ void gemv1_accumulate(const uint4 (&w)[RT][CPL], const uint32_t (&act)[MT][CPL][16],
                                                 int KV, int lane, int (&part)[RT][MT]) {
  int acc[RT][MT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[r][m][j] = 0;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    if (i == CPL - 1 && lane + 32 * i >= KV) break;   // only the last chunk slot can be empty
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const uint32_t wd[4] = {w[r][i].x, w[r][i].y, w[r][i].z, w[r][i].w};
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t e = wd[g] & (0x03030303u << (2 * j));
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[r][m][j] = dp4a_us(e, act[m][i][4 * g + j], acc[r][m][j]);
        }
    }
  }
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m)
      part[r][m] = acc[r][m][0] + (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) + (acc[r][m][3] >> 6);
}

// Warp-wide sum of the partials (one redux per row and token), correction and
// rescale, store.
template <int MT, int RT>
__device__ __forceinline__ void gemv1_finish(const int (&part)[RT][MT], int tile, int N, int lane, const int (&R)[MT],
                                             const float (&f)[MT], void* __restrict__ Y, int out_mode,
                                             const float* __restrict__ bias = nullptr) {
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int tot = __reduce_add_sync(0xffffffffu, part[r][m]);
      const int n = tile * RT + r;
      if (lane == r * MT + m && n < N) {
        const int a = tot - R[m];
        const size_t o = static_cast<size_t>(m) * N + n;
        if (out_mode == kOutI32) {
          static_cast<int*>(Y)[o] = a;
        } else {
          float y = __fmul_rn(__int2float_rn(a), f[m]);
          if (bias) y = __fadd_rn(y, __ldg(bias + n));
          if (out_mode == kOutF32)
            static_cast<float*>(Y)[o] = y;
          else
            static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
        }
      }
    }
}

template <int MT, int CPL, int RT, int D, int THREADS, int MINB>
__global__ void __launch_bounds__(THREADS, MINB)
    bl_decode_rows_kernel(const void* __restrict__ X, int x_is_i8, int K, int N, const uint4* __restrict__ Wp,
                 const float* __restrict__ gamma_p, int Q, void* __restrict__ Y, int out_mode, int tiles_per_cta) {
  constexpr int WARPS = THREADS / 32;
  __shared__ __align__(16) uint8_t s_act[MT][8192];
  __shared__ __align__(16) uint32_t s_red_f[MT][WARPS];
  __shared__ int s_red_i[MT][WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KV = K >> 6;
  const int ntiles = (N + RT - 1) / RT;
  const int tbeg = blockIdx.x * tiles_per_cta;
  const int tend = min(ntiles, tbeg + tiles_per_cta);

  // 1. stream this CTA's weight rows into L2; dependent-launch handshake
  if (threadIdx.x == 0 && tbeg < tend) {
    const size_t row_bytes = static_cast<size_t>(K) >> 2;
    const size_t r0 = static_cast<size_t>(tbeg) * RT;
    const size_t r1 = min(static_cast<size_t>(N), static_cast<size_t>(tend) * RT);
    const char* base = reinterpret_cast<const char*>(Wp) + r0 * row_bytes;
    const size_t bytes = (r1 - r0) * row_bytes;
    for (size_t off = 0; off < bytes; off += kPrefetchChunk)
      bulk_prefetch_l2(base + off, static_cast<uint32_t>(min(static_cast<size_t>(kPrefetchChunk), bytes - off)));
  }
  pdl_launch_dependents();
  pdl_wait();

  // token loads first, then the first D weight tiles of this warp (a ring of
  // D register buffers, refilled as tiles are consumed)
  constexpr int U = (8192 / 8 + THREADS - 1) / THREADS;   // 16-byte token loads per thread
  const int nch = x_is_i8 ? (K >> 4) : (K >> 3);
  uint4 xv[MT][U];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + THREADS * u;
      xv[m][u] = (c < nch) ? __ldg(static_cast<const uint4*>(X) + static_cast<size_t>(m) * nch + c)
                           : make_uint4(0, 0, 0, 0);
    }
  uint4 wr[D][RT][CPL];
#pragma unroll
  for (int d = 0; d < D; ++d) gemv1_load<CPL, RT>(wr[d], Wp, tbeg + warp + d * WARPS, tend, N, KV, lane);
  const float gamma = (out_mode == kOutI32) ? 1.f : __ldg(gamma_p);

  // 2. the CTA quantises the token(s) into s_act (plain byte order)
  int rsum[MT];
  float s[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    rsum[m] = 0;
    s[m] = 1.f;
  }
  if (!x_is_i8) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) amax = fmaxf(amax, absmax8_bf16(xv[m][u]));
      // non-negative floats order like their bit patterns
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      if (lane == 0) s_red_f[m][warp] = wmax;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint32_t bmax = 0;
#pragma unroll
      for (int w = 0; w < WARPS; w += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(&s_red_f[m][w]);
        bmax = max(bmax, max(max(v.x, v.y), max(v.z, v.w)));
      }
      s[m] = __fdiv_rn(static_cast<float>(Q), fmaxf(__uint_as_float(bmax), 1e-5f));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = threadIdx.x + THREADS * u;
        if (c < nch) *reinterpret_cast<uint2*>(&s_act[m][act_swz(8u * c)]) = quant8_bf16(xv[m][u], s[m], rsum[m]);
      }
    }
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = threadIdx.x + THREADS * u;
        if (c < nch) {
          const uint4 v = xv[m][u];
          rsum[m] = __dp4a(static_cast<int>(v.x), 0x01010101, rsum[m]);
          rsum[m] = __dp4a(static_cast<int>(v.y), 0x01010101, rsum[m]);
          rsum[m] = __dp4a(static_cast<int>(v.z), 0x01010101, rsum[m]);
          rsum[m] = __dp4a(static_cast<int>(v.w), 0x01010101, rsum[m]);
          *reinterpret_cast<uint4*>(&s_act[m][act_swz(16u * c)]) = v;
        }
      }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int ws = __reduce_add_sync(0xffffffffu, rsum[m]);
    if (lane == 0) s_red_i[m][warp] = ws;
  }
  __syncthreads();
  int R[MT];
  float f[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    R[m] = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) R[m] += s_red_i[m][w];
    f[m] = (x_is_i8 || out_mode == kOutI32) ? 0.f : __fdiv_rn(gamma, s[m]);
  }

  // this lane's activation chunks, kept in registers
  uint32_t act[MT][CPL][16];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int c = lane + 32 * i;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (c < KV) v = *reinterpret_cast<const uint4*>(&s_act[m][act_swz(64u * c + 16u * g)]);
        act[m][i][4 * g + 0] = v.x;
        act[m][i][4 * g + 1] = v.y;
        act[m][i][4 * g + 2] = v.z;
        act[m][i][4 * g + 3] = v.w;
      }
    }

  // 3.-5. this warp's tiles tbeg + warp + k*WARPS; ring buffer d holds tile k
  // with k % D == d.  A round accumulates its D tiles together (independent
  // chains), refills the ring with the next round's loads, then reduces and
  // stores while those loads are in flight.
  for (int t = tbeg + warp; t < tend; t += D * WARPS) {
    int part[D][RT][MT];
#pragma unroll
    for (int d = 0; d < D; ++d) gemv1_accumulate<MT, CPL, RT>(wr[d], act, KV, lane, part[d]);
#pragma unroll
    for (int d = 0; d < D; ++d) gemv1_load<CPL, RT>(wr[d], Wp, t + (d + D) * WARPS, tend, N, KV, lane);
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (t + d * WARPS < tend) gemv1_finish<MT, RT>(part[d], t + d * WARPS, N, lane, R, f, Y, out_mode);
  }
}


// ---------------------------------------------------------------------------
// Launch table of the one-token decode kernel (bl_decode.cuh): one launch can
// serve several independent one-token problems; CTAs [cta_begin, cta_begin +
// ctas) of the grid work on problem i.
// ---------------------------------------------------------------------------
struct G2Problem {
  const void* X;
  const void* U;      // squared-ReLU gated mode: the up projection's output;
                      // RMSNorm mode: the norm's bf16 weight [K] or null (else unused)
  const uint8_t* Wp;
  const float* gamma;
  void* Y;
  int K;
  int N;
  int rows_per_cta;   // decode kernel: q = N / ctas; CTA c takes q + (c < rem) rows
  int cta_begin;      // first CTA of this problem in the launch
  int ctas;           // CTAs of this problem
  int rows_rem;       // rem = N % ctas
  const float* bias;  // optional fp32 [N] added after the rescale
  float eps;          // RMSNorm mode: added to the mean of squares
  int chunk_rows;     // decode kernel: rows per bulk copy (a multiple of the row group)
  int slots;          // decode kernel: chunks the ring holds at once
  int ksplit;         // decode kernel: warps that split one row (resident 2-bit rows)
};
constexpr int kG2MaxProblems = 8;
struct G2Table {
  G2Problem p[kG2MaxProblems];
  int count;
};

}  // namespace bl
