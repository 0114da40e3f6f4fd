// One-token BitLinear forward (decode).
//
// What it computes is the one-token case of the BitLinear forward of "BitNet
// b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear" (absmean ternary weights, eq. (1);
// per-token absmax int8 activations, eq. (2); integer matmul and one rescale,
// eq. (3)): y = f32(f32(sum_k c*q) * f32(gamma/s)), the sum taken exactly in
// integers (each ternary weight adds, subtracts or skips an activation: the
// same page, section "Why 1.58 Bits? The Power of Zero").
//
// Every weight byte is read once and the token is 5-16 KB, so the work is a
// stream of weight rows through the SMs.  One launch serves a table of
// independent one-token problems with any mix of K (e.g. the up, gate and
// down projections of a feed-forward block); the host gives each problem
// CTAs by a cost model, one CTA per SM.  Ring modes:
//
//   * row-lane (2-bit layers of a few MB, the usual case): a CTA takes a
//     little under half an SM (a 96 KB ring plus the token codes, <= 56
//     registers a thread), so the CTAs of the next launch on the stream
//     (programmatic dependent launch, triggered at the start) become
//     resident beside this launch's CTAs and fetch their weights while this
//     launch runs.  Rows sit in the ring at a padded stride and each lane
//     owns whole rows (see the row-lane consumer loop);
//   * resident, column-split (the same footprint; rows of more than 512 a
//     CTA, and base-3 rows): lane l takes 32-bit words l, l + 32, ... of
//     every row, with its columns' token codes in registers (base-3 rows:
//     read from shared memory);
//   * big (layers of tens of MB): 2-bit rows with 8 consumer warps and a
//     96 KB ring, two CTAs per SM (base-3 rows: 16 warps, a 192 KB ring, one
//     CTA per SM), column-split with a lane's 16-byte chunks' token codes in
//     registers.
//
// In all of them a producer warp copies the CTA's row range into the ring
// (cp.async.bulk, one mbarrier per chunk) BEFORE the dependency wait: the
// weights and gamma are parameters, not produced by the preceding kernel.
// The consumer warps wait for the token and quantise it once per CTA into
// shared memory.  Then:
//
//   * 2-bit rows: per 32-bit word four masked unsigned-by-signed dp4a (slice
//     j of a word holds 4^j * (c+1) in each byte) into four accumulators,
//     folded exactly as acc0 + acc1/4 + acc2/16 + acc3/64;
//   * base-3 rows: five digits a byte, recovered by tripling (see dec3_dot);
//   * the stored digits are c + 1, so sum_k c*q = sum_k (c+1)*q - sum_k q:
//     each partial sum starts at minus the sum of the codes of the columns
//     it covers (per lane in the column-split modes, per 256-column block in
//     row-lane mode), so the totals are the exact dot products;
//   * column-split: one warp reduction per row, then lane r of the group
//     rescales and stores row r; row-lane: shared row totals and one store
//     pass per CTA.
#pragma once

#include <type_traits>

#include "bl_act.cuh"
#include "bl_gemv.cuh"
#include "bl_norm.cuh"
#include "bl_weights.cuh"

namespace bl {

constexpr int kDecWarps = 16;                        // consumer warps (+ one producer warp)
constexpr int kDecMaxSlots = 16;
constexpr int kDecMaxK = 8192;
constexpr int kDecRegMaxWpl = 5;                     // resident register path: K <= 2560
// token codes, plus zero codes under the padding digits of a base-3 row
constexpr int kDecActBytes = kDecMaxK + 128;
// resident mode: two CTAs per SM
constexpr int kDecRingBytes = 96 * 1024;
constexpr int kDecChunkMax = 32 * 1024;
// big mode, 2-bit rows: 8 consumer warps and a 96 KB ring, so that two CTAs
// fit on an SM and the next launch's CTA fetches its first chunks while the
// current one streams; base-3 rows (more instructions a byte) keep 16 warps
// and a 192 KB ring, one CTA per SM
constexpr int kDecBigWarps = 8;
constexpr int kDecBigRingBytes = 96 * 1024;
constexpr int kDecBigChunkMax = 32 * 1024;
constexpr int kDecB3BigRingBytes = 192 * 1024;
constexpr int kDecB3BigChunkMax = 64 * 1024;
constexpr int kDecBigMaxCpl = kDecMaxK / 2048;       // 16-byte chunks a lane

// Launch shape of a (mode, format) pair.
__host__ __device__ constexpr bool dec_big2(int mode, int fmt) { return mode == 1 && fmt == 0; }
__host__ __device__ constexpr int dec_warps(int mode, int fmt) { return dec_big2(mode, fmt) ? kDecBigWarps : kDecWarps; }
__host__ __device__ constexpr int dec_threads(int mode, int fmt) { return (dec_warps(mode, fmt) + 1) * 32; }
__host__ __device__ constexpr int dec_ring_bytes(int mode, int fmt) {
  return mode != 1 ? kDecRingBytes : (fmt == 0 ? kDecBigRingBytes : kDecB3BigRingBytes);
}
__host__ __device__ constexpr int dec_chunk_max(int mode, int fmt) {
  return mode != 1 ? kDecChunkMax : (fmt == 0 ? kDecBigChunkMax : kDecB3BigChunkMax);
}
__host__ __device__ constexpr int dec_smem_bytes(int mode, int fmt) { return dec_ring_bytes(mode, fmt) + kDecActBytes; }

// What the token prologue forms before the quantisation: nothing (bf16
// activations or int8 codes), the squared-ReLU input, or the RMS- or
// layer-normalised token.  A template parameter so that the plain path
// carries no code for the others.
enum DecPre : int { kDecPlain = 0, kDecRelu2 = 1, kDecRms = 2, kDecLn = 3 };
// Weight storage: 2 bits a weight, or base 3 (five weights a byte, see
// bl_weights.cuh).
enum DecFmt : int { kFmt2Bit = 0, kFmtBase3 = 1 };
// kModeRowLane: resident layers of 2-bit rows with each lane owning a whole
// row (see the consumer loop); kModeResident keeps the column-split register
// path for row ranges that this mode does not take.
enum DecMode : int { kModeResident = 0, kModeBig = 1, kModeRowLane = 2 };

// Row-lane mode: rows of a 32-row tile sit in shared memory at a stride of an
// odd number of 16-byte units (the row's bytes plus 16 or 32), so the eight
// lanes of a quarter-warp that read the same 16-byte column of eight rows hit
// eight different bank groups; a tile is one ring chunk.
constexpr int kDecLaneRows = 32;
constexpr int kDecLaneMaxRows = 512;             // rows of one CTA (shared row totals)
constexpr int kDecLaneMaxRT = 2;                 // rows a lane takes at once (measured best of 1, 2, 4)
constexpr int kDecHalfSegs = kDecMaxK / 256;     // 256-weight (four-column) items of the longest row
__host__ __device__ constexpr int dec_lane_stride(int row_bytes) {
  return row_bytes + (((row_bytes >> 4) & 1) ? 32 : 16);
}

// Rows a warp (or a team of warps) takes at once.
constexpr int kDecRegRows = 2;     // 2-bit rows, token codes in registers
constexpr int kDecB3Rows = 4;      // base-3 rows, resident mode
constexpr int kDecBigRows = 2;     // big mode (both formats)
// Largest team of warps that splits one long row (resident 2-bit rows), and
// the most rows a chunk of split rows may hold (the rows' shared totals).
constexpr int kDecMaxSplit = 8;
constexpr int kDecSplitRows = 256;

template <int FMT, int MODE>
__host__ __device__ constexpr int dec_group_rows() {
  return MODE == kModeBig ? kDecBigRows : (FMT == kFmt2Bit ? kDecRegRows : kDecB3Rows);
}

// Output conversion known at compile time (bf16, the forward's output) or
// chosen at run time (the fp32 and int32 test exports).
constexpr int kOutAny = -1;

// ---------------------------------------------------------------------------
// token quantisation helpers
// ---------------------------------------------------------------------------

// Eight codes without their sum (the register path forms it per lane).
__device__ __forceinline__ uint2 dec_quant8(uint4 v, float s) {
  return make_uint2(codes4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y), s),
                    codes4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w), s));
}

__device__ __forceinline__ uint2 dec_quant8_f32(const float (&h)[8], float s) {
  return make_uint2(codes4(h[0], h[1], h[2], h[3], s), codes4(h[4], h[5], h[6], h[7], s));
}

// minus the sum of the int8 codes in four words (four independent chains)
__device__ __forceinline__ void dec_negsum4(uint4 v, int (&r)[4]) {
  r[0] = __dp4a(static_cast<int>(v.x), -1, r[0]);
  r[1] = __dp4a(static_cast<int>(v.y), -1, r[1]);
  r[2] = __dp4a(static_cast<int>(v.z), -1, r[2]);
  r[3] = __dp4a(static_cast<int>(v.w), -1, r[3]);
}

// ---------------------------------------------------------------------------
// per-group work
// ---------------------------------------------------------------------------

// Rescale and store one output: y = f32(f32(acc) * f) (+ bias), as bf16 or
// fp32, or the accumulator itself.
template <int OUT>
__device__ __forceinline__ void dec_put(int t, int n, float f, void* __restrict__ Y, const float* __restrict__ bias,
                                        int out_mode) {
  const int om = OUT == kOutAny ? out_mode : OUT;
  if (om == kOutI32) {
    static_cast<int*>(Y)[n] = t;
  } else {
    float y = __fmul_rn(__int2float_rn(t), f);
    if (bias) y = __fadd_rn(y, __ldg(bias + n));
    if (om == kOutF32)
      static_cast<float*>(Y)[n] = y;
    else
      static_cast<__nv_bfloat16*>(Y)[n] = __float2bfloat16_rn(y);
  }
}

// Warp sum of each row's partial: the total of row r in lane r.
template <int RT>
__device__ __forceinline__ int dec_warp_totals(const int (&part)[RT], int lane) {
  int t = __reduce_add_sync(0xffffffffu, part[0]);
#pragma unroll
  for (int r = 1; r < RT; ++r) {
    const int tr = __reduce_add_sync(0xffffffffu, part[r]);
    t = lane == r ? tr : t;
  }
  return t;
}

__device__ __forceinline__ int dec_fold(const int (&a)[4]) { return a[0] + (a[1] >> 2) + (a[2] >> 4) + (a[3] >> 6); }

// 2-bit rows, resident mode: lane l takes words word0 + l + 32 i (i < WPL)
// of RT rows at rowp (rows past nlive read row 0 again and are discarded);
// act holds the token's codes of those words (zero past the end of the row
// or of the lane's part of it, so the weight words read there, still inside
// the CTA's shared memory, contribute nothing).
template <int RT, int WPL>
__device__ __forceinline__ void dec_dot_reg(const uint8_t* rowp, int row_bytes, int nlive, int word0, int lane,
                                            const uint32_t (&act)[WPL][4], int neg_r, int (&part)[RT]) {
  const uint32_t* p[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r)
    p[r] = reinterpret_cast<const uint32_t*>(rowp + (r < nlive ? r : 0) * row_bytes) + word0 + lane;
  int acc[RT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    acc[r][0] = neg_r;
    acc[r][1] = acc[r][2] = acc[r][3] = 0;
  }
#pragma unroll
  for (int i = 0; i < WPL; ++i) {
    uint32_t w[RT];
#pragma unroll
    for (int r = 0; r < RT; ++r) w[r] = p[r][32 * i];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int r = 0; r < RT; ++r) acc[r][j] = dp4a_us(w[r] & (0x03030303u << (2 * j)), act[i][j], acc[r][j]);
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) part[r] = dec_fold(acc[r]);
}

// 2-bit rows, big mode: lane l takes the 16-byte chunks l + 32 i (i < CPL,
// 64 weights each) of RT rows; act[4 i + g] holds the token's codes of word g
// of chunk i (zero past the end of the row).
template <int RT, int CPL>
__device__ __forceinline__ void dec_dot_big(const uint8_t* rowp, int row_bytes, int nlive, int lane,
                                            const uint32_t (&act)[4 * CPL][4], int neg_r, int (&part)[RT]) {
  const uint4* p[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) p[r] = reinterpret_cast<const uint4*>(rowp + (r < nlive ? r : 0) * row_bytes) + lane;
  int acc[RT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    acc[r][0] = neg_r;
    acc[r][1] = acc[r][2] = acc[r][3] = 0;
  }
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    uint32_t w[RT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const uint4 v = p[r][32 * i];
      w[r][0] = v.x;
      w[r][1] = v.y;
      w[r][2] = v.z;
      w[r][3] = v.w;
    }
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int r = 0; r < RT; ++r)
          acc[r][j] = dp4a_us(w[r][g] & (0x03030303u << (2 * j)), act[4 * i + g][j], acc[r][j]);
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) part[r] = dec_fold(acc[r]);
}

// Base-3 rows: lane l takes the 32-bit words l, l+32, ... of each row (20
// weights each).  The even and odd bytes of a word sit in two registers as
// 16-bit lanes; tripling a lane moves the next digit into its high byte
// (digit = (3x) >> 8, exact because 3^5 = 243 < 256), one byte permute
// gathers the four digits of a level into the byte lanes of one register
// (weights k = 20g + 4L .. +3, consecutive), and one unsigned x signed dp4a
// takes it with the four matching codes.
template <int RT>
__device__ __forceinline__ void dec3_dot(const uint8_t* rowp, int row_bytes, int nlive, int rwords, int lane,
                                         const uint8_t* s_act, int neg_r, int (&part)[RT]) {
  const uint32_t* p[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) p[r] = reinterpret_cast<const uint32_t*>(rowp + (r < nlive ? r : 0) * row_bytes);
  int acc[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) acc[r] = neg_r;
#pragma unroll 2
  for (int wi = lane; wi < rwords; wi += 32) {
    const uint32_t* a = reinterpret_cast<const uint32_t*>(s_act + 20 * wi);
    uint32_t av[5];
#pragma unroll
    for (int L = 0; L < 5; ++L) av[L] = a[L];
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const uint32_t w = p[r][wi];
      uint32_t e = w & 0x00ff00ffu, o = (w >> 8) & 0x00ff00ffu;
#pragma unroll
      for (int L = 0; L < 5; ++L) {
        const uint32_t e3 = e * 3u, o3 = o * 3u;
        acc[r] = dp4a_us(__byte_perm(e3, o3, 0x7351), av[L], acc[r]);
        e = e3 & 0x00ff00ffu;
        o = o3 & 0x00ff00ffu;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) part[r] = acc[r];
}

// Row-lane mode, one item: lane l takes rows l + 32 j (j < RT) of the rows
// at row0 (stride rstride; rows at or past `live` read row 0 again and are
// discarded), nu <= 4 16-byte columns from row0 on, with the token codes of
// those columns at ap (16 bytes per 32-bit weight word); each row starts at
// neg (minus the codes' sum) and its folded total is added to rs[row].
template <int RT>
__device__ __forceinline__ void dec_lane_item(const uint8_t* row0, int rstride, int live, int lane, const uint4* ap,
                                              int nu, int neg, int* rs) {
  const uint4* wp[RT];
#pragma unroll
  for (int j = 0; j < RT; ++j) {
    const int r = 32 * j + lane;
    wp[j] = reinterpret_cast<const uint4*>(row0 + (r < live ? r : 0) * rstride);
  }
  int acc[RT][4];
#pragma unroll
  for (int j = 0; j < RT; ++j) {
    acc[j][0] = neg;
    acc[j][1] = acc[j][2] = acc[j][3] = 0;
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    if (t < nu) {
      uint32_t w[RT][4];
#pragma unroll
      for (int j = 0; j < RT; ++j) {
        const uint4 v = wp[j][t];
        w[j][0] = v.x;
        w[j][1] = v.y;
        w[j][2] = v.z;
        w[j][3] = v.w;
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint4 a = ap[4 * t + g];
#pragma unroll
        for (int j = 0; j < RT; ++j) {
          acc[j][0] = dp4a_us(w[j][g] & 0x03030303u, a.x, acc[j][0]);
          acc[j][1] = dp4a_us(w[j][g] & 0x0c0c0c0cu, a.y, acc[j][1]);
          acc[j][2] = dp4a_us(w[j][g] & 0x30303030u, a.z, acc[j][2]);
          acc[j][3] = dp4a_us(w[j][g] & 0xc0c0c0c0u, a.w, acc[j][3]);
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < RT; ++j) {
    const int r = 32 * j + lane;
    if (r < live) atomicAdd(rs + r, dec_fold(acc[j]));
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

// A: resident mode, the register path's words per lane (0: none; a problem
// takes it when ceil(K / 512) == A); big mode with 2-bit rows, 16-byte chunks
// per lane (ceil(K / 2048) of at most A for every problem of the launch).
template <int A, int PRE, int FMT, int MODE>
__global__ void __launch_bounds__(dec_threads(MODE, FMT), (MODE == kModeBig && FMT == kFmtBase3) ? 1 : 2)
    bl_decode_kernel(const __grid_constant__ G2Table tab, int in_mode, int Q, int out_mode,
                     unsigned long long limit_ns) {
  constexpr int CW = dec_warps(MODE, FMT);
  constexpr bool RELU2 = PRE == kDecRelu2;
  constexpr bool RMS = PRE == kDecRms;
  constexpr bool LN = PRE == kDecLn;
  constexpr bool NORM = RMS || LN;
  constexpr bool B3 = FMT == kFmtBase3;
  constexpr bool BIG = MODE == kModeBig;
  constexpr bool LANES = MODE == kModeRowLane;
  constexpr int RING = dec_ring_bytes(MODE, FMT);
  static_assert(!B3 || (A == 0 && PRE == kDecPlain), "base-3 rows take the shared-memory token path");
  static_assert(!LANES || (A == 0 && !B3), "row-lane mode: 2-bit rows, token codes read from shared memory");
  static_assert(!BIG || B3 || (A >= 1 && A <= kDecBigMaxCpl), "big mode keeps 1..4 chunks a lane");
  static_assert(B3 || BIG || LANES || (A >= 1 && A <= kDecRegMaxWpl), "resident register path: 1..5 words a lane");
  int pi = 0;
  while (pi + 1 < tab.count && static_cast<int>(blockIdx.x) >= tab.p[pi + 1].cta_begin) ++pi;
  const void* __restrict__ X = tab.p[pi].X;
  const void* __restrict__ Up = tab.p[pi].U;
  const uint8_t* __restrict__ Wp = tab.p[pi].Wp;
  const float* __restrict__ gamma_p = tab.p[pi].gamma;
  void* __restrict__ Y = tab.p[pi].Y;
  const float* __restrict__ bias = tab.p[pi].bias;
  const int K = tab.p[pi].K;
  const int CR = tab.p[pi].chunk_rows, slots = tab.p[pi].slots;
  const int cta = static_cast<int>(blockIdx.x) - tab.p[pi].cta_begin;
  // rows [r0, r0 + rows): q or q + 1 rows a CTA, the first `rem` CTAs one more
  const int q_rows = tab.p[pi].rows_per_cta, rem = tab.p[pi].rows_rem;
  const int r0 = cta * q_rows + min(cta, rem);
  const int rows = q_rows + (cta < rem ? 1 : 0);

  extern __shared__ __align__(128) uint8_t dec_smem[];
  uint8_t* const s_act = dec_smem + RING;
  static_assert(CW % 4 == 0, "partials are read four at a time");
  __shared__ __align__(16) uint32_t s_red_f[CW];
  __shared__ __align__(8) uint64_t full[kDecMaxSlots], empty[kDecMaxSlots];
  __shared__ int abort_flag;
  __shared__ unsigned long long s_sq[NORM ? kSqLimbs : 1];
  __shared__ unsigned long long s_win[NORM ? 2 * CW : 1];
  __shared__ uint32_t s_dig[RMS ? kSqLimbs : 1];
  __shared__ unsigned long long s_s1[LN ? kS1Limbs : 1];
  __shared__ long long s_w1[LN ? CW : 1];
  __shared__ float s_rms, s_mu;
  // row totals of split rows (resident register path: two chunks' worth;
  // row-lane mode: one per row of the CTA), and minus the sum of the token's
  // codes in each 512-weight segment (row-lane mode)
  __shared__ int s_rowsum[kDecLaneMaxRows];
  __shared__ int s_negseg[LANES ? kDecHalfSegs : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = B3 ? base3_row_words(K) : (K >> 4);   // 32-bit words of a row
  const int row_bytes = 4 * words;
  const int nch = rows > 0 ? (rows + CR - 1) / CR : 0;
  // row-lane mode: rows at a padded stride in the ring
  const int rstride = LANES ? dec_lane_stride(row_bytes) : row_bytes;
  const int chunk_bytes = CR * rstride;
  volatile int* abort_v = &abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (NORM) {
    if (threadIdx.x < kSqLimbs) s_sq[threadIdx.x] = 0ull;
  }
  if constexpr (LN) {
    if (threadIdx.x < kS1Limbs) s_s1[threadIdx.x] = 0ull;
  }
  if constexpr (LANES) {
    for (int t = threadIdx.x; t < kDecLaneMaxRows; t += blockDim.x) s_rowsum[t] = 0;
    if (threadIdx.x < kDecHalfSegs) s_negseg[threadIdx.x] = 0;
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == CW && LANES) {
    // ---------------- producer, row-lane mode: one copy per row, padded stride ----------------
    const uint8_t* base = Wp + static_cast<size_t>(r0) * row_bytes;
    const int pre = min(nch, slots);
    if (lane == 0)
      for (int c = 0; c < pre; ++c)
        mbar_arrive_expect_tx(&full[c], static_cast<uint32_t>(min(CR, rows - c * CR) * row_bytes));
    __syncwarp();
    for (int c = 0; c < pre; ++c) {
      const int cr = min(CR, rows - c * CR);
      for (int r = lane; r < cr; r += 32)
        bulk_load(dec_smem + c * chunk_bytes + r * rstride, base + static_cast<size_t>(c * CR + r) * row_bytes,
                  static_cast<uint32_t>(row_bytes), &full[c]);
    }
    if (lane == 0 && nch > pre) {
      const size_t off0 = static_cast<size_t>(pre) * CR * row_bytes;
      const size_t bytes = static_cast<size_t>(rows) * row_bytes;
      for (size_t off = off0; off < bytes; off += kPrefetchChunk)
        bulk_prefetch_l2(base + off, static_cast<uint32_t>(min(static_cast<size_t>(kPrefetchChunk), bytes - off)));
    }
    int issued = pre;
    int s = 0, ph = 1;   // slot and phase parity of chunk c
    for (int c = pre; c < nch; ++c) {
      const int cr = min(CR, rows - c * CR);
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&empty[s], ph ^ 1u, abort_v, limit_ns, 21);
        if (ok) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(cr * row_bytes));
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int r = lane; r < cr; r += 32)
        bulk_load(dec_smem + s * chunk_bytes + r * rstride, base + static_cast<size_t>(c * CR + r) * row_bytes,
                  static_cast<uint32_t>(row_bytes), &full[s]);
      issued = c + 1;
      if (++s == slots) {
        s = 0;
        ph ^= 1;
      }
    }
    // no copy may be in flight when the CTA exits
    if (lane == 0)
      for (int s = 0; s < slots && s < issued; ++s) {
        const int last = s + slots * ((issued - 1 - s) / slots);
        mbar_wait(&full[s], (last / slots) & 1, nullptr, limit_ns, 22);
      }
    return;
  }
  if (warp == CW) {
    // ---------------- producer (never waits on the preceding kernel) ----------------
    if (lane == 0) {
      const uint8_t* base = Wp + static_cast<size_t>(r0) * row_bytes;
      const int pre = min(nch, slots);
      for (int c = 0; c < pre; ++c) {
        const uint32_t bytes = static_cast<uint32_t>(min(CR, rows - c * CR) * row_bytes);
        mbar_arrive_expect_tx(&full[c], bytes);
        bulk_load(dec_smem + c * chunk_bytes, base + static_cast<size_t>(c) * chunk_bytes, bytes, &full[c]);
      }
      // the rest of this CTA's rows: towards L2 now, in resident mode (small
      // layers: it is all fetched during the previous launch).  Big mode
      // leaves it to the ring: a prefetch of every CTA's whole range would
      // queue the first chunks and the token behind tens of MB.
      if (!BIG && nch > pre) {
        const size_t off0 = static_cast<size_t>(pre) * chunk_bytes;
        const size_t bytes = static_cast<size_t>(rows) * row_bytes;
        for (size_t off = off0; off < bytes; off += kPrefetchChunk)
          bulk_prefetch_l2(base + off, static_cast<uint32_t>(min(static_cast<size_t>(kPrefetchChunk), bytes - off)));
      }
      int issued = pre;
      // chunk c = pre (only when pre == slots) reuses slot 0 in its second phase
      int s = 0, ph = 1;   // slot and phase parity of chunk c
      for (int c = pre; c < nch; ++c) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_v, limit_ns, 21)) break;
        const uint32_t bytes = static_cast<uint32_t>(min(CR, rows - c * CR) * row_bytes);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(dec_smem + s * chunk_bytes, base + static_cast<size_t>(c) * chunk_bytes, bytes, &full[s]);
        issued = c + 1;
        if (++s == slots) {
          s = 0;
          ph ^= 1;
        }
      }
      // no copy may be in flight when the CTA exits
      for (int s = 0; s < slots && s < issued; ++s) {
        const int last = s + slots * ((issued - 1 - s) / slots);
        mbar_wait(&full[s], (last / slots) & 1, nullptr, limit_ns, 22);
      }
    }
    return;
  }

  // ---------------- consumers: parameters first, then the token ----------------
  constexpr int CT = CW * 32;
  constexpr int U = (kDecMaxK / 8 + CT - 1) / CT;
  const float gamma = (out_mode == kOutI32) ? 1.f : __ldg(gamma_p);
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
  const bool gated = RELU2 && in_mode == kInRelu2Gated;
  const int nchx = x_is_i8 ? (K >> 4) : (K >> 3);
  uint4 xv[U], uv[RELU2 ? U : 1];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = threadIdx.x + CT * u;
    xv[u] = (c < nchx) ? __ldg(static_cast<const uint4*>(X) + c) : make_uint4(0, 0, 0, 0);
    if constexpr (RELU2) uv[u] = (gated && c < nchx) ? __ldg(static_cast<const uint4*>(Up) + c) : make_uint4(0, 0, 0, 0);
  }
  if constexpr (NORM) {
    // exact mean of squares (RMSNorm) or exact mean and variance
    // (LayerNorm): register windows anchored at the token's largest
    // exponent, far values in shared limb counters; then the normalised
    // bf16 token in place of the input
    float xmax = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (threadIdx.x + CT * u < nchx) xmax = fmaxf(xmax, absmax8_bf16(xv[u]));
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
    const float thr = norm_thr(E);
    unsigned long long lo = 0ull, hi = 0ull;
    long long w1 = 0ll;
    double p1 = 0.0, p2 = 0.0;
    static_assert(8 * U <= kNormFlush, "one flush per thread");
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (threadIdx.x + CT * u < nchx) norm_add8<LN>(xv[u], E, thr, p1, p2, w1, lo, hi, s_s1, s_sq);
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
    named_bar_sync(1, CT);
    if (warp == 0) {
      if constexpr (LN) {
        float mu, var;
        ln_block_stats(s_w1, s_win, CW, E, s_s1, s_sq, static_cast<uint32_t>(K), lane, mu, var);
        if (lane == 0) {
          s_mu = mu;
          s_rms = __fsqrt_rn(__fadd_rn(var, tab.p[pi].eps));
        }
      } else {
        const float ms = sq_block_mean(s_win, CW, E, s_sq, s_dig, static_cast<uint32_t>(K), lane);
        if (lane == 0) s_rms = __fsqrt_rn(__fadd_rn(ms, tab.p[pi].eps));
      }
    }
    named_bar_sync(1, CT);
    const float r = s_rms;
    if constexpr (LN) {
      const float mu = s_mu;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (threadIdx.x + CT * u < nchx) xv[u] = ln_apply8(xv[u], mu, r);
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (threadIdx.x + CT * u < nchx) xv[u] = rms_apply8(xv[u], nw[u], has_nw, r);
    }
  }
  float sc = 1.f;
  if (!x_is_i8) {
    uint32_t am;
    if constexpr (RELU2) {
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float h[8];
        relu2_8(xv[u], uv[u], gated, h);
        amax = fmaxf(amax, absmax8_f32(h));
      }
      am = __float_as_uint(amax);
    } else {
      uint32_t a2 = 0u;   // chunks past the row end are zero
#pragma unroll
      for (int u = 0; u < U; ++u) a2 = __vmaxu2(a2, absmax2_bf16x8(xv[u]));
      am = max(a2 & 0xffffu, a2 >> 16) << 16;   // bf16 bits -> fp32 bits
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, am);
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
      uint2 q = make_uint2(0u, 0u);
      if (c < nchx) {
        if constexpr (RELU2) {
          float h[8];
          relu2_8(xv[u], uv[u], gated, h);
          q = dec_quant8_f32(h, sc);
        } else {
          q = dec_quant8(xv[u], sc);
        }
        *reinterpret_cast<uint2*>(&s_act[8 * c]) = q;
      }
      if constexpr (LANES) {
        // the warp's 256 codes are one four-column item's
        const int ns = __reduce_add_sync(0xffffffffu, __dp4a(static_cast<int>(q.x), -1, __dp4a(static_cast<int>(q.y), -1, 0)));
        if (lane == 0 && c - lane < nchx) atomicAdd(&s_negseg[(c - lane) >> 5], ns);
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + CT * u;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (c < nchx) {
        v = xv[u];
        *reinterpret_cast<uint4*>(&s_act[16 * c]) = v;
      }
      if constexpr (LANES) {
        // each half-warp's 256 codes are one four-column item's
        int r4[4] = {0, 0, 0, 0};
        dec_negsum4(v, r4);
        int ns = (r4[0] + r4[1]) + (r4[2] + r4[3]);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) ns += __shfl_xor_sync(0xffffffffu, ns, o);
        const int c0 = c - (lane & 15);
        if ((lane & 15) == 0 && c0 < nchx) atomicAdd(&s_negseg[c0 >> 4], ns);
      }
    }
  }
  if constexpr (B3) {
    // codes under the padding digits of the row's last words are zero
    for (int k = K + threadIdx.x * 4; k < 20 * words; k += CT * 4) *reinterpret_cast<uint32_t*>(&s_act[k]) = 0u;
  }
  const float f = (x_is_i8 || out_mode == kOutI32) ? 0.f : __fdiv_rn(gamma, sc);
  named_bar_sync(1, CT);

  // ---------------- consumers: this lane's token codes ----------------
  // 2-bit rows take the register path: resident mode, a team of S warps
  // splits each row into S parts of 32 * A words (S = 1 for rows of at most
  // 32 * A words) and lane l of part p keeps the codes of words
  // 32 A p + l + 32 i (i < A); big mode, lane l keeps the codes of the 16-byte
  // chunks l + 32 i (i < A), word g of chunk i at [4 i + g].  Base-3 rows read
  // the codes from shared memory.
  constexpr bool REGP = !B3 && !LANES;
  const int S = (BIG || LANES) ? 1 : tab.p[pi].ksplit;
  const int team = warp / S, part = warp - team * S, teams = CW / S;
  const int word0 = BIG ? 0 : 32 * A * part;
  constexpr int AW = (B3 || LANES) ? 1 : (BIG ? 4 * A : A);
  uint32_t act[AW][4];
  int nr[4] = {0, 0, 0, 0};
  if constexpr (REGP) {
#pragma unroll
    for (int i = 0; i < AW; ++i) {
      const int wi = BIG ? 4 * (lane + 32 * (i / 4)) + (i % 4) : word0 + lane + 32 * i;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (wi < words) v = *reinterpret_cast<const uint4*>(&s_act[16 * wi]);
      act[i][0] = v.x;
      act[i][1] = v.y;
      act[i][2] = v.z;
      act[i][3] = v.w;
      dec_negsum4(v, nr);
    }
  } else if constexpr (B3) {
    for (int wi = lane; wi < words; wi += 32) {
      const uint32_t* a = reinterpret_cast<const uint32_t*>(&s_act[20 * wi]);
      dec_negsum4(make_uint4(a[0], a[1], a[2], a[3]), nr);
      nr[0] = __dp4a(static_cast<int>(a[4]), -1, nr[0]);
    }
  }
  const int neg_r = (nr[0] + nr[1]) + (nr[2] + nr[3]);

  // ---------------- consumers: row groups, chunk by chunk ----------------
  // group g holds rows [g*RT, g*RT + RT) of this CTA's range and goes to team
  // g % teams; chunks hold a multiple of RT rows, so a group never straddles
  // two.  Rows split across a team (S > 1): each part adds its row totals
  // into shared row sums (integer adds, in any order) and the consumers store
  // the rows after meeting once at the end, when the CTA has at most
  // kDecSplitRows rows; otherwise once per chunk (chunks of split rows hold
  // at most kDecSplitRows rows), with the chunk waits agreed CTA-wide so a
  // timeout unwinds every consumer together.
  if constexpr (LANES) {
    // ---------------- consumers, row-lane mode ----------------
    // Lane l of a warp owns rows l, l + 32, ... of a group of up to 128 rows
    // (one to four 32-row ring chunks) and takes four 16-byte columns (256
    // weights) of them per item: per column, its rows' 16 bytes (the eight
    // lanes of a quarter-warp hit eight bank groups thanks to the padded
    // stride) and the matching 64 token codes (one address for the whole
    // warp, shared by the lane's rows), four masked dp4a per 32-bit word.
    // Item i goes to warp i % 16.  Each item adds its rows' partial totals
    // into shared row totals (integer adds, any order); one store pass ends
    // the CTA.  When the ring must be reused, chunks are taken one at a time
    // (one row a lane) and released in order.
    const int upr = K >> 6;               // 16-byte columns of a row
    const int nhs = (upr + 3) >> 2;       // four-column items of a row
    const uint4* act4 = reinterpret_cast<const uint4*>(s_act);
    if (nch <= slots) {
      // every chunk resident: row r at r * rstride
      constexpr int GR = kDecLaneRows * kDecLaneMaxRT;   // rows of a group
      const int ngroups = (rows + GR - 1) / GR;
      for (int it = warp; it < ngroups * nhs; it += CW) {
        const int g = it / nhs, h = it - g * nhs;
        const int live = rows - GR * g;
        const int rt = min(kDecLaneMaxRT, (live + 31) >> 5);
        bool ok = true;
        for (int j = 0; j < rt; ++j) ok = ok && mbar_wait(&full[kDecLaneMaxRT * g + j], 0, abort_v, limit_ns, 23);
        if (!__all_sync(0xffffffffu, ok)) break;
        const uint8_t* row0 = dec_smem + static_cast<size_t>(GR * g) * rstride + 64 * h;
        const uint4* ap = act4 + 16 * h;
        const int nu = min(4, upr - 4 * h);
        const int neg = s_negseg[h];
        int* rs = s_rowsum + GR * g;
        if (kDecLaneMaxRT >= 4 && rt == 4)
          dec_lane_item<(kDecLaneMaxRT >= 4 ? 4 : 1)>(row0, rstride, live, lane, ap, nu, neg, rs);
        else if (kDecLaneMaxRT >= 3 && rt == 3)
          dec_lane_item<(kDecLaneMaxRT >= 3 ? 3 : 1)>(row0, rstride, live, lane, ap, nu, neg, rs);
        else if (kDecLaneMaxRT >= 2 && rt == 2)
          dec_lane_item<(kDecLaneMaxRT >= 2 ? 2 : 1)>(row0, rstride, live, lane, ap, nu, neg, rs);
        else
          dec_lane_item<1>(row0, rstride, live, lane, ap, nu, neg, rs);
      }
    } else {
      int it = warp, ibase = 0;
      int s = 0, ph = 0;
      for (int c = 0; c < nch; ++c) {
        bool ok = mbar_wait(&full[s], ph, abort_v, limit_ns, 23);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const int c0 = c * CR;
        const uint8_t* sbase = dec_smem + s * chunk_bytes;
        for (; it < ibase + nhs; it += CW) {
          const int h = it - ibase;
          dec_lane_item<1>(sbase + 64 * h, rstride, min(CR, rows - c0), lane, act4 + 16 * h, min(4, upr - 4 * h),
                           s_negseg[h], s_rowsum + c0);
        }
        ibase += nhs;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == slots) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    // every consumer leaves the loop (a bounded wait that gives up ends it
    // too), so all of them reach this barrier; a stalled CTA stores nothing
    const bool all_ok = named_bar_and(1, CT, !*abort_v);
    if (all_ok)
      for (int t = threadIdx.x; t < rows; t += CT) dec_put<kOutAny>(s_rowsum[t], r0 + t, f, Y, bias, out_mode);
    return;
  }
  constexpr int RT = dec_group_rows<FMT, MODE>();
  const bool active = team < teams;
  const bool once = rows <= kDecSplitRows;   // split rows: one final store pass
  if (S > 1) {
    for (int t = threadIdx.x; t < 2 * kDecSplitRows; t += CT) s_rowsum[t] = 0;
    named_bar_sync(1, CT);
  }
  auto walk = [&](auto out_tag) {
    constexpr int OUT = decltype(out_tag)::value;
    int g = team;
    int s = 0, ph = 0;   // ring slot and phase parity of chunk c
    // The previous group's row totals wait here (lane r: row r) and are
    // stored after the next group's dot products are issued: the warp
    // reductions and the store's dependent chain then overlap the next
    // group's work instead of stalling the warp.
    int pend_t = 0, pend_row = 0, pend_n = 0;   // pend_n: live rows (0: none)
    int* pend_rs = nullptr;
    auto flush = [&]() {
      if (lane < pend_n) {
        if (S == 1)
          dec_put<OUT>(pend_t, r0 + pend_row + lane, f, Y, bias, out_mode);
        else
          atomicAdd(pend_rs + lane, pend_t);
      }
    };
    for (int c = 0; c < nch; ++c) {
      bool ok = mbar_wait(&full[s], ph, abort_v, limit_ns, 23);
      ok = __all_sync(0xffffffffu, ok);
      if (S > 1 && !once) ok = named_bar_and(1, CT, ok);
      if (!ok) break;
      const int c0 = c * CR;
      const int cend = min(c0 + CR, rows);
      const uint8_t* sbase = dec_smem + s * chunk_bytes;
      // split rows: row r of the CTA at rs[r - rbase]
      int* rs = once ? s_rowsum : s_rowsum + (c & 1) * kDecSplitRows;
      const int rbase = once ? 0 : c0;
      if (active) {
        for (; g * RT < cend; g += teams) {
          const int lr = g * RT;
          const int nlive = min(RT, rows - lr);
          const uint8_t* rowp = sbase + (lr - c0) * row_bytes;
          int pt[RT];
          if constexpr (B3) {
            dec3_dot<RT>(rowp, row_bytes, nlive, words, lane, s_act, neg_r, pt);
          } else if constexpr (BIG) {
            dec_dot_big<RT, A>(rowp, row_bytes, nlive, lane, act, neg_r, pt);
          } else {
            dec_dot_reg<RT, AW>(rowp, row_bytes, nlive, word0, lane, act, neg_r, pt);
          }
          const int t = dec_warp_totals<RT>(pt, lane);
          flush();
          pend_t = t;
          pend_row = lr;
          pend_n = nlive;
          pend_rs = rs + (lr - rbase);
        }
      }
      if (S > 1 && !once) {
        // every part of the chunk's rows has added its totals: store them,
        // and clear the buffer for chunk c + 2 (its adds follow the next
        // chunk's agreement barrier)
        flush();
        pend_n = 0;
        named_bar_sync(1, CT);
        for (int t = threadIdx.x; t < cend - c0; t += CT) {
          dec_put<OUT>(rs[t], r0 + c0 + t, f, Y, bias, out_mode);
          rs[t] = 0;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == slots) {
        s = 0;
        ph ^= 1;
      }
    }
    flush();
    if (S > 1 && once) {
      // every consumer leaves the loop (a bounded wait that gives up ends it
      // too), so all of them reach this barrier; a stalled CTA stores
      // nothing (its status word records the timeout)
      const bool all_ok = named_bar_and(1, CT, !*abort_v);
      if (all_ok)
        for (int t = threadIdx.x; t < rows; t += CT) dec_put<OUT>(s_rowsum[t], r0 + t, f, Y, bias, out_mode);
    }
  };
  // one copy of the loop for every output type: a smaller kernel runs faster
  // here than one specialised for bf16 (instruction fetch)
  walk(std::integral_constant<int, kOutAny>{});
}

}  // namespace bl
