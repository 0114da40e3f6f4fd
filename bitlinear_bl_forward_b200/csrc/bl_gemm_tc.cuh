// Prefill / batched path: ternary x int8 GEMM on the 5th-generation tensor
// cores (tcgen05.mma kind::i8, int32 accumulation in tensor memory).
//
// "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "The
// Mathematical Formulation of BitLinear", eq. (3): Y = (X~ . W~^T) *
// (gamma / scale_X).  "BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs",
// section "1. Hybrid W1.58 / A4 Quantization Function": integer dot products
// accumulated in 32-bit registers.
//
// Tile: 128 weight rows (the MMA's M, one TMEM lane per output feature) x BN
// tokens (the MMA's N).  D[n, m] = sum_k A[n, k] * B[m, k] with
//   A = stored codes u = c + 1 in {0, 1, 2}, expanded to int8 straight into
//       tensor memory (never into shared memory), and
//   B = int8 activation codes, TMA-loaded into shared memory with the
//       128-byte swizzle the MMA descriptor names;
// the epilogue subtracts R[m] = sum_k q[m, k] to undo the +1 offset, then
// applies f_m = gamma / s_m.
//
// Warp roles (192 threads):
//   warp 0     TMA producer: per 128-wide K stage, one packed-weight box
//              [128 rows x 32 bytes] (32-byte swizzle) and one activation box
//              [BN rows x 128 bytes] (128-byte swizzle) onto one mbarrier;
//   warp 1     owns the TMEM allocation; one thread issues 4 MMAs (K = 32
//              each) per stage and commits them to the stage's "empty"
//              barrier, finally to the accumulator barrier;
//   warps 2-5  expanders then epilogue: thread = weight row (TMEM lane); per
//              stage it reads its row's 32 packed bytes, turns each 32-bit
//              word into four int8x4 columns with shift+mask and stores 32
//              columns with tcgen05.st; after the last MMA it reads its row
//              of D with tcgen05.ld and writes the outputs.
//
// Every wait is bounded (see mbar_wait): a stalled pipeline records
// BL_ERR_TIMEOUT, drains the copies it issued, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "bl_common.cuh"
#include "bl_gemv.cuh"

namespace bl {

constexpr int kTcThreads = 192;
constexpr int kTcRows = 128;      // weight rows per CTA (MMA M)
constexpr int kTcBK = 128;        // K per pipeline stage
constexpr int kTcStages = 4;
constexpr int kTcWStageBytes = kTcRows * kTcBK / 4;   // 4 KB packed

// debug flag: the producer issues no copies, so every consumer wait runs out
constexpr int kDebugSkipLoads = 1;

// wait-site identifiers recorded with a timeout
enum : unsigned int {
  kSiteProdEmpty = 1,
  kSiteExpFull = 2,
  kSiteExpEmpty = 3,
  kSiteMmaExfull = 4,
  kSiteAcc = 5,
  kSiteDrain = 6,
  kSiteSelftest = 0xEE
};

template <int BN>
struct TcCfg {
  static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "unsupported token tile");
  static constexpr int kXStageBytes = BN * kTcBK;
  static constexpr int kACol = (BN <= 128) ? 128 : 256;        // first TMEM column of the A stages
  static constexpr int kTmemCols = (kACol + 32 * kTcStages <= 256) ? 256 : 512;
  static constexpr int kBarOffset = kTcStages * (kXStageBytes + kTcWStageBytes);
  static constexpr int kBarBytes = (3 * kTcStages + 1) * 8 + 16;
  static constexpr int kEpiOffset = kBarOffset + kBarBytes;
  static constexpr int kUsedBytes = kEpiOffset + BN * 8;
  // pad the request so at most 2 CTAs (256-column TMEM) or 1 CTA (512) share an SM
  static constexpr int kMinBytes = (kTmemCols == 512) ? 120 * 1024 : 100 * 1024;
  static constexpr int kSmemBytes = (kUsedBytes > kMinBytes ? kUsedBytes : kMinBytes) + 1024;
};

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int M, int N,
                   int K, const int* __restrict__ Rg, const float* __restrict__ sg, const float* __restrict__ gamma_p,
                   void* __restrict__ Y, int out_mode, unsigned long long limit_ns, int debug_flags) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sW = smem + kTcStages * C::kXStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + kTcStages;
  uint64_t* exfull = empty + kTcStages;
  uint64_t* accfull = exfull + kTcStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* sR = reinterpret_cast<int*>(smem + C::kEpiOffset);
  float* sF = reinterpret_cast<float*>(sR + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcRows, m0 = blockIdx.y * BN;
  const int nk = (K + kTcBK - 1) / kTcBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&exfull[s], 128);
    }
    mbar_init(accfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {
    for (int j = threadIdx.x - 64; j < BN; j += 128) {
      const int m = m0 + j;
      int r = 0;
      float f = 0.f;
      if (m < M) {
        r = Rg[m];
        if (out_mode != kOutI32) f = __fdiv_rn(*gamma_p, sg[m]);
      }
      sR[j] = r;
      sF[j] = f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmW);
      int nissued = 0;
      if (!(debug_flags & kDebugSkipLoads)) {
        for (int ks = 0; ks < nk; ++ks) {
          const int s = ks % kTcStages;
          const uint32_t ph = (ks / kTcStages) & 1;
          if (ks >= kTcStages && !mbar_wait(&empty[s], ph ^ 1u, abort_flag, limit_ns, kSiteProdEmpty)) break;
          mbar_arrive_expect_tx(&full[s], C::kXStageBytes + kTcWStageBytes);
          tma_load_2d(sX + s * C::kXStageBytes, &tmX, ks * kTcBK, m0, &full[s]);
          tma_load_2d(sW + s * kTcWStageBytes, &tmW, ks * (kTcBK / 4), n0, &full[s]);
          nissued = ks + 1;
        }
      }
      // every copy issued into this CTA's shared memory must land before exit
      for (int s = 0; s < kTcStages && s < nissued; ++s) {
        const int last = s + kTcStages * ((nissued - 1 - s) / kTcStages);
        mbar_wait(&full[s], (last / kTcStages) & 1, nullptr, limit_ns, kSiteDrain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(kTcRows, BN);
      for (int ks = 0; ks < nk; ++ks) {
        const int s = ks % kTcStages;
        const uint32_t ph = (ks / kTcStages) & 1;
        if (!mbar_wait(&exfull[s], ph, abort_flag, limit_ns, kSiteMmaExfull)) break;
        tc_fence_after();
        const uint32_t xs = smem_u32(sX + s * C::kXStageBytes);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 32; ++kk) {
          const uint32_t a_tmem = tmem + C::kACol + 32 * s + 8 * kk;
          const uint64_t bdesc = smem_desc_k_sw128(xs + 32 * kk);
          mma_i8_ts(tmem, a_tmem, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      // always commit, and wait here, so no MMA is in flight when TMEM is freed
      tc_commit(accfull);
      mbar_wait(accfull, 0, nullptr, limit_ns, kSiteAcc);
    }
  } else {
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int r = q * 32 + lane;             // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t wsw = static_cast<uint32_t>((r >> 2) & 1) << 4;   // 32-byte swizzle of the packed box
    for (int ks = 0; ks < nk; ++ks) {
      const int s = ks % kTcStages;
      const uint32_t ph = (ks / kTcStages) & 1;
      bool ok = mbar_wait(&full[s], ph, abort_flag, limit_ns, kSiteExpFull);
      if (ok && ks >= kTcStages) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, limit_ns, kSiteExpEmpty);
      // tcgen05.st is warp-collective: the whole warp goes on or stops together
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t wrow = smem_u32(sW + s * kTcWStageBytes) + r * 32;
      const uint4 lo = ld_shared_v4(wrow + (0u ^ wsw));
      const uint4 hi = ld_shared_v4(wrow + (16u ^ wsw));
      const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
      uint32_t v[32];
#pragma unroll
      for (int g = 0; g < 8; ++g)
#pragma unroll
        for (int j = 0; j < 4; ++j) v[4 * g + j] = (wd[g] >> (2 * j)) & 0x03030303u;
      tmem_st_32x32b_x32(tmem + lane_base + C::kACol + 32 * s, v);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&exfull[s]);
    }
    // epilogue
    const bool acc_ok = mbar_wait(accfull, 0, abort_flag, limit_ns, kSiteAcc) && !*abort_flag;
    if (__all_sync(0xffffffffu, acc_ok)) {
      tc_fence_after();
      const int n = n0 + r;
      constexpr int kChunk = BN < 32 ? BN : 32;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += kChunk) {
        uint32_t v[32];
        if constexpr (kChunk == 32)
          tmem_ld_32x32b_x32(tmem + lane_base + c0, v);
        else
          tmem_ld_32x32b_x16(tmem + lane_base + c0, v);
        tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            const int m = m0 + c0 + t;
            if (m < M) {
              const int a = static_cast<int>(v[t]) - sR[c0 + t];
              const size_t o = static_cast<size_t>(m) * N + n;
              if (out_mode == kOutI32) {
                static_cast<int*>(Y)[o] = a;
              } else {
                const float y = __fmul_rn(__int2float_rn(a), sF[c0 + t]);
                if (out_mode == kOutF32)
                  static_cast<float*>(Y)[o] = y;
                else
                  static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives at; the wait must give up after limit_ns and record a timeout.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, int* out) {
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
