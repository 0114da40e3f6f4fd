// Persistent tensor-core GEMM for few tokens (M <= 64).
//
// The BitLinear matmul and rescale ("BitNet b1.58: The 1-Bit Ternary LLM
// Architecture Guide", section "The Mathematical Formulation of BitLinear",
// eq. (3)): D[n, m] = sum_k u[n, k] * q[m, k] on tcgen05.mma kind::i8 with the
// expanded weight codes u = c + 1 as the A operand in tensor memory and the
// int8 activation codes as the B operand in shared memory; the epilogue
// subtracts R[m] = sum_k q[m, k] and applies f_m = gamma / s_m.
//
// One CTA per SM walks a static list of tiles (128 weight rows x BN tokens),
// token tiles fastest so the CTAs of a wave share weight tiles through L2.
// A pipeline stage covers K = 512: the packed weight tile is 128 rows of 128
// contiguous bytes (one 128-byte-swizzled TMA box: whole 128-byte row
// segments from DRAM), the tokens four 128-byte boxes.  With few tokens an
// MMA (M = 128, N <= 64, K = 32) is short (about 46 cycles, measured), so the
// fixed costs around it decide the speed: each hand-off between roles moves a
// whole stage (16 MMAs), and one commit per stage frees both the shared
// memory stage and, three stages later, the tensor-memory slot.
// Rings:
//   smem ring (S stages):  TMA producer -> expanders (packed W) and MMA (X);
//                          freed by the MMA's commit to empty[s];
//   TMEM A ring (3 slots of 128 columns, one stage each): expanders
//                          (tcgen05.st of int8 codes) -> MMA; slot reuse waits
//                          on the empty[] phase of the stage that last used it;
//   accumulators (2):      MMA -> epilogue; freed by the epilogue warps,
//                          so tile i's epilogue overlaps tile i+1's MMAs.
// Warps: 0 producer, 1 MMA issuer (owns TMEM), then EXPG groups of four
// expander warps (group e takes the stages g with g % EXPG == e), then four
// epilogue warps.
// Every wait is bounded; a stalled pipeline records BL_ERR_TIMEOUT, each
// role unwinds, the producer drains its copies, the MMA thread waits for its
// MMAs, and TMEM is freed before the CTA exits.
#pragma once

#include <cuda_bf16.h>

#include "bl_common.cuh"
#include "bl_tc_common.cuh"
#include "bl_gemv.cuh"

namespace bl {

constexpr int kP2ASlots = 3;                     // tensor-memory A slots, one K = 512 stage each
constexpr int kP2Sub = 4;                        // sub-stages of K = 128 per stage
constexpr int kP2BK = kTcBK * kP2Sub;            // K per stage (512)
constexpr int kP2WStageBytes = kTcRows * kP2BK / 4;   // 16 KB packed
constexpr int kP2ASlotCols = kP2BK / 4;               // 128 columns of int8x4 per slot
// warps: producer, MMA issuer, EXPG groups of 4 expander warps, 4 epilogue warps
template <int EXPG>
struct P2Warps {
  static constexpr int kFirstExp = 2;
  static constexpr int kFirstEpi = 2 + 4 * EXPG;
  static constexpr int kThreads = 32 * (kFirstEpi + 4);
};
constexpr int kP2SmemBudget = 200 * 1024;

template <int BN>
struct P2Cfg {
  static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128, "unsupported token tile");
  static constexpr int kXSubBytes = BN * kTcBK;               // one 128-byte-wide token box
  static constexpr int kXStageBytes = kP2Sub * kXSubBytes;
  static constexpr int kStageBytes = kXStageBytes + kP2WStageBytes;
  static constexpr int kStagesRaw = kP2SmemBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 24 ? 24 : kStagesRaw;
  static constexpr int kAccCols = BN < 32 ? 32 : BN;             // per accumulator buffer
  static constexpr int kACol = 2 * kAccCols;                      // first TMEM column of the A ring
  static constexpr int kTmemCols = 512;
  static_assert(kACol + kP2ASlotCols * kP2ASlots <= 512, "accumulators and A slots exceed tensor memory");
  static constexpr int kBarOffset = kStages * kStageBytes;
  // barriers: full[S], empty[S], afull[slots], accfull[2], accempty[2], drain
  static constexpr int kNumBars = 2 * kStages + kP2ASlots + 5;
  static constexpr int kEpiOffset = kBarOffset + kNumBars * 8 + 16;
  static constexpr int kUsedBytes = kEpiOffset + 2 * BN * 8;
  static constexpr int kSmemBytes = kUsedBytes + 1024;
};

template <int BN, int EXPG>
__global__ void __launch_bounds__(P2Warps<EXPG>::kThreads, 1)
    bl_mma_persistent_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int M,
                              int N, int K, const int* __restrict__ Rg, const float* __restrict__ sg,
                              const float* __restrict__ gamma_p, void* __restrict__ Y, int out_mode,
                              const float* __restrict__ bias, unsigned long long limit_ns) {
  using C = P2Cfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sW = smem + S * C::kXStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;
  uint64_t* accfull = afull + kP2ASlots;
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* sR = reinterpret_cast<int*>(smem + C::kEpiOffset);   // [2][BN]
  float* sF = reinterpret_cast<float*>(sR + 2 * BN);        // [2][BN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (K + kP2BK - 1) / kP2BK;   // stages per tile (K beyond the end reads zeros)
  const int mt = (M + BN - 1) / BN;
  const int ntiles = mt * ((N + kTcRows - 1) / kTcRows);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int t = 0; t < kP2ASlots; ++t) {
      mbar_init(&afull[t], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmW);
      uint32_t g = 0;   // global k-stage counter across tiles
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
        const int m0 = (tile % mt) * BN, n0 = (tile / mt) * kTcRows;
        for (int ks = 0; ks < nk; ++ks, ++g) {
          const int s = g % S;
          if (g >= static_cast<uint32_t>(S) &&
              !mbar_wait(&empty[s], ((g / S) & 1) ^ 1u, abort_flag, limit_ns, kSiteProdEmpty)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          tma_load_2d(sW + s * kP2WStageBytes, &tmW, ks * (kP2BK / 4), n0, &full[s]);
#pragma unroll
          for (int j = 0; j < kP2Sub; ++j)
            tma_load_2d(sX + s * C::kXStageBytes + j * C::kXSubBytes, &tmX, ks * kP2BK + j * kTcBK, m0, &full[s]);
        }
      }
      // every copy issued into this CTA's shared memory must land before exit
      const uint32_t issued = g;
      for (uint32_t s = 0; s < static_cast<uint32_t>(S) && s < issued; ++s) {
        const uint32_t last = s + S * ((issued - 1 - s) / S);
        mbar_wait(&full[s], (last / S) & 1, nullptr, limit_ns, kSiteDrain);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(kTcRows, BN);
      // ring positions kept as counters: this thread's instruction count
      // bounds the MMA rate
      const uint32_t dlo0 = desc_sw128_lo(smem_u32(sX));
      int s = 0, t = 0;
      uint32_t tph = 0;   // phase parity of afull[t]
      int i = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x, ++i) {
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(&accempty[b], ((i >> 1) & 1) ^ 1u, abort_flag, limit_ns, kSiteAcc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + b * C::kAccCols;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(&afull[t], tph, abort_flag, limit_ns, kSiteMmaExfull)) {
            stop = true;
            break;
          }
          tc_fence_after();
          // the stage's 16 MMAs (K = 32 each) from one asm block: MMA k reads
          // A column 8k of the slot and token box k / 4, bytes 32 (k % 4)
          static_assert(kP2Sub * (kTcBK / 32) == 16, "one stage is sixteen MMAs");
          mma_i8_stage16<C::kXSubBytes / 16>(d_tmem, tmem + C::kACol + kP2ASlotCols * t,
                                             dlo0 + s * (C::kXStageBytes / 16), kDescSw128Hi, idesc,
                                             ks != 0 ? 1u : 0u);
          // one commit frees both the smem stage (producer) and, three stages
          // later, the tensor-memory slot (expanders wait on the same phase)
          tc_commit(&empty[s]);
          if (++s == S) s = 0;
          if (++t == kP2ASlots) {
            t = 0;
            tph ^= 1u;
          }
        }
        if (stop) break;
        tc_commit(&accfull[b]);
      }
      // no MMA may be in flight when TMEM is freed
      tc_commit(drain);
      mbar_wait(drain, 0, nullptr, limit_ns, kSiteDrain);
    }
  } else if (warp < P2Warps<EXPG>::kFirstEpi) {
    // ---------------- expanders: packed W (smem) -> int8 codes (TMEM) ----------------
    const int grp = (warp - P2Warps<EXPG>::kFirstExp) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t rsw = static_cast<uint32_t>(r & 7);   // 128-byte swizzle: 16-byte chunk c sits at c ^ (r % 8)
    uint32_t g = 0;   // stage counter
    bool stop = false;
    for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
      for (int ks = 0; ks < nk; ++ks, ++g) {
        if (static_cast<int>(g % EXPG) != grp) continue;
        const int s = g % S;
        const int t = g % kP2ASlots;
        bool ok = mbar_wait(&full[s], (g / S) & 1, abort_flag, limit_ns, kSiteExpFull);
        // slot t was last read by the MMAs of stage g - kP2ASlots, whose commit
        // completes that stage's phase of empty[]; no later phase of that
        // barrier can complete before this stage is expanded
        if (ok && g >= static_cast<uint32_t>(kP2ASlots)) {
          const uint32_t prev = g - kP2ASlots;
          ok = mbar_wait(&empty[prev % S], (prev / S) & 1, abort_flag, limit_ns, kSiteExpEmpty);
        }
        if (!__all_sync(0xffffffffu, ok)) {
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t wrow = smem_u32(sW + s * kP2WStageBytes) + r * 128;
        // four sub-steps of K = 128 (32 bytes of the row each); one wait for all stores
#pragma unroll 1
        for (uint32_t j = 0; j < kP2Sub; ++j) {
          const uint4 lo = ld_shared_v4(wrow + (((2u * j + 0u) ^ rsw) << 4));
          const uint4 hi = ld_shared_v4(wrow + (((2u * j + 1u) ^ rsw) << 4));
          const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          uint32_t v[32];
#pragma unroll
          for (int gw = 0; gw < 8; ++gw)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) v[4 * gw + jj] = (wd[gw] >> (2 * jj)) & 0x03030303u;
          tmem_st_32x32b_x32(tmem + lane_base + C::kACol + kP2ASlotCols * t + 32 * j, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&afull[t]);
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int et = threadIdx.x - 32 * P2Warps<EXPG>::kFirstEpi;   // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float gamma = (out_mode == kOutI32) ? 1.f : *gamma_p;
    int i = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int b = i & 1;
      const int m0 = (tile % mt) * BN, n0 = (tile / mt) * kTcRows;
      // per-token constants of this tile into smem buffer b
      for (int j = et; j < BN; j += 128) {
        const int m = m0 + j;
        int rv = 0;
        float fv = 0.f;
        if (m < M) {
          rv = Rg[m];
          if (out_mode != kOutI32) fv = __fdiv_rn(gamma, sg[m]);
        }
        sR[b * BN + j] = rv;
        sF[b * BN + j] = fv;
      }
      __syncwarp();
      named_bar_sync(2, 128);
      const bool ok = mbar_wait(&accfull[b], (i >> 1) & 1, abort_flag, limit_ns, kSiteAcc) && !*abort_flag;
      // the four epilogue warps decide together (they share named barriers)
      __syncwarp();
      if (!named_bar_and(3, 128, ok)) break;
      tc_fence_after();
      const int n = n0 + r;
      const float bias_n = (bias && n < N) ? __ldg(bias + n) : 0.f;
      constexpr int kChunk = BN < 32 ? BN : 32;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += kChunk) {
        uint32_t v[32];
        if constexpr (kChunk == 32)
          tmem_ld_32x32b_x32(tmem + lane_base + b * C::kAccCols + c0, v);
        else
          tmem_ld_32x32b_x16(tmem + lane_base + b * C::kAccCols + c0, v);
        tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            const int m = m0 + c0 + t;
            if (m < M) {
              const int a = static_cast<int>(v[t]) - sR[b * BN + c0 + t];
              const size_t o = static_cast<size_t>(m) * N + n;
              if (out_mode == kOutI32) {
                static_cast<int*>(Y)[o] = a;
              } else {
                float y = __fmul_rn(__int2float_rn(a), sF[b * BN + c0 + t]);
                if (bias) y = __fadd_rn(y, bias_n);
                if (out_mode == kOutF32)
                  static_cast<float*>(Y)[o] = y;
                else
                  static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[b]);
      __syncwarp();
      named_bar_sync(2, 128);   // sR/sF buffer b is rewritten two tiles later
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

}  // namespace bl
