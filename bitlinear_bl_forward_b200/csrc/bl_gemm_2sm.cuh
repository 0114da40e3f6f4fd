// Persistent tensor-core GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same arithmetic as the other tensor-core kernels ("BitNet b1.58: The 1-Bit
// Ternary LLM Architecture Guide", section "The Mathematical Formulation of
// BitLinear", eq. (3)): D[n, m] = sum_k u[n, k] * q[m, k] with u = c + 1 the
// expanded weight codes (A, tensor memory) and q the int8 activation codes
// (B, shared memory); the epilogue subtracts R[m] and applies gamma / s_m.
//
// A cluster of two CTAs (two SMs) computes one 256 x BN tile per MMA
// (M = 256 weight rows, N = BN tokens):
//   * each CTA stages its own 128 weight rows (packed) and HALF of the token
//     tile (BN/2 rows of int8 codes) in its own shared memory with TMA, and
//     expands its weight rows into its own tensor memory;
//   * the leader CTA (rank 0) issues tcgen05.mma.cta_group::2; the pair's
//     tensor cores share the two halves of B, so each SM loads and serves only
//     half of the activation tile -- the traffic that bounds the one-SM
//     kernel;
//   * the leader's tcgen05.commit arrives on the barriers of both CTAs
//     (smem stage free, TMEM A slot free, accumulator full); the peer's
//     expanders and epilogue warps arrive on the leader's barriers remotely.
// Rings: S shared-memory stages of K = 512 (16 MMAs per hand-off: a commit
// costs about as much pipe time as two short MMAs, so fewer hand-offs), two
// TMEM A slots of 128 columns (a slot is free again once the stage that last
// used it is done), 2 accumulators (the epilogue of tile i overlaps the MMAs
// of i+1).
// Warps: 0 producer, 1 MMA issuer (leader) / TMEM owner, 2-5 expanders,
// 6-13 epilogue (two per TMEM lane quadrant, 64 tokens each: the epilogue of
// a tile must finish within the next tile's main loop, which for K = 2560 is
// only ten stages).  All waits are bounded; the pair meets at a cluster barrier
// before TMEM is freed, after the leader has waited for its last MMA.
#pragma once

#include <cuda_bf16.h>

#include "bl_common.cuh"
#include "bl_tc_common.cuh"
#include "bl_gemv.cuh"

namespace bl {

// warps: 0 producer, 1 MMA issuer, 2..(2+4*kQExpGroups-1) expanders (group e
// expands the stages g with g % kQExpGroups == e), then 4 epilogue warps
constexpr int kQExpGroups = 1;   // measured: a second group does not help
constexpr int kQFirstEpi = 2 + 4 * kQExpGroups;
constexpr int kQEpiWarps = 8;   // two per TMEM lane quadrant, each takes half of the tile's tokens
constexpr int kQThreads = 32 * (kQFirstEpi + kQEpiWarps);
constexpr int kQBK = 512;                       // K per pipeline stage: kQBK / 32 MMAs per hand-off
constexpr int kQASlots = 2;                     // TMEM: 2 x 128 accumulator + 2 A slots = 512 columns
constexpr int kQASlotCols = kQBK / 4;           // int8 codes, 4 per 32-bit column
constexpr int kQBN = 128;                       // tokens per pair tile (MMA N)
constexpr int kQHalf = kQBN / 2;                // token rows staged per CTA
constexpr int kQRows = 256;                     // weight rows per pair tile (MMA M)
constexpr int kQXBoxBytes = kQHalf * 128;       // one 128-byte-wide activation box (SW128)
constexpr int kQXStageBytes = kQHalf * kQBK;    // 16 KB: kQBK / 128 boxes
constexpr int kQWRowBytes = kQBK / 4;           // packed bytes of a weight row per stage
constexpr int kQWStageBytes = kTcRows * kQWRowBytes;   // 128-byte rows (SW128)
constexpr int kQStageBytes = kQXStageBytes + kQWStageBytes;
constexpr int kQStages = 3;                    // 144 KB
constexpr int kQEpiCols = kQBN / 2;             // tokens per epilogue warp
constexpr int kQStageOutBytes = kQEpiCols * 32 * 2;  // bf16 [64 tokens][32 rows] per epilogue warp
constexpr int kQAccCols = kQBN;
constexpr int kQACol = 2 * kQAccCols;
constexpr int kQTmemCols = 512;
constexpr int kQOutOffset = kQStages * kQStageBytes;
constexpr int kQBarOffset = kQOutOffset + kQEpiWarps * kQStageOutBytes;
// barriers: full[S], done[S] (stage consumed by the MMAs: frees its shared
// memory and, kQASlots stages later, its TMEM A slot), afull[4], accfull[2],
// accempty[2], drain
constexpr int kQNumBars = 2 * kQStages + kQASlots + 5;
constexpr int kQEpiOffset = kQBarOffset + kQNumBars * 8 + 16;
constexpr int kQSmemBytes = kQEpiOffset + 2 * kQBN * 8 + 1024;

// One weight tensor of a launch.  A launch serves one or two problems that
// share the quantised activations (e.g. the up and gate projections of a
// feed-forward block): its tiles run over the weight rows of problem 0 then
// of problem 1, so every activation tile is quantised once and each tile of
// either weight tensor is computed by the same pipeline.
struct QOut {
  CUtensorMap tmW;      // packed weights [N, K/4] (128-byte swizzle boxes)
  CUtensorMap tmY;      // bf16 output [M, N] (TMA stores), when tma_store
  const float* gamma;   // device fp32
  void* Y;              // output [M, N]
  const float* bias;    // optional fp32 [N]
  int N;
  int tma_store;
  int ntn;              // weight-row tiles: ceil(N / 256)
};
struct QProblems {
  QOut p[2];
  int count;
};

__global__ void __launch_bounds__(kQThreads, 1)
    bl_mma_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ QProblems P, int M, int K,
                        const int* __restrict__ Rg, const float* __restrict__ sg, int out_mode,
                        unsigned long long limit_ns) {
  constexpr int S = kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sW = smem + S * kQXStageBytes;
  static_assert(2 * kQAccCols + kQASlots * kQASlotCols <= kQTmemCols, "tensor memory budget");
  uint8_t* sOut = smem + kQOutOffset;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQBarOffset);
  uint64_t* done = full + S;
  uint64_t* afull = done + S;         // leader's copy counts both CTAs' expander warps
  uint64_t* accfull = afull + kQASlots;
  uint64_t* accempty = accfull + 2;   // leader's copy counts both CTAs' epilogue threads
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* sR = reinterpret_cast<int*>(smem + kQEpiOffset);   // [2][BN]
  float* sF = reinterpret_cast<float*>(sR + 2 * kQBN);    // [2][BN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nk = (K + kQBK - 1) / kQBK;
  const int mt = (M + kQBN - 1) / kQBN;
  const int ntn0 = P.p[0].ntn;
  const int ntiles = mt * (ntn0 + (P.count > 1 ? P.p[1].ntn : 0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], 1);
    }
    for (int t = 0; t < kQASlots; ++t) mbar_init(&afull[t], 8);   // one arrival per expander warp of each CTA
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 2 * 32 * kQEpiWarps);   // every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kQTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&P.p[0].tmW);
      if (P.count > 1) prefetch_tmap(&P.p[1].tmW);
      uint32_t g = 0;
      bool stop = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
        const int m0 = (tile % mt) * kQBN + static_cast<int>(rank) * kQHalf;
        const int nt = tile / mt, w = nt >= ntn0 ? 1 : 0;
        const int n0 = (nt - (w ? ntn0 : 0)) * kQRows + static_cast<int>(rank) * kTcRows;
        const CUtensorMap* tmW = &P.p[w].tmW;
        for (int ks = 0; ks < nk; ++ks, ++g) {
          const int s = g % S;
          if (g >= static_cast<uint32_t>(S) &&
              !mbar_wait_cluster(&done[s], ((g / S) & 1) ^ 1u, abort_flag, limit_ns, kSiteProdEmpty)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kQStageBytes);
#pragma unroll
          for (int bx = 0; bx < kQBK / 128; ++bx)
            tma_load_2d(sX + s * kQXStageBytes + bx * kQXBoxBytes, &tmX, ks * kQBK + bx * 128, m0, &full[s]);
          tma_load_2d(sW + s * kQWStageBytes, tmW, ks * (kQBK / 4), n0, &full[s]);
        }
      }
      const uint32_t issued = g;
      for (uint32_t s = 0; s < static_cast<uint32_t>(S) && s < issued; ++s) {
        const uint32_t last = s + S * ((issued - 1 - s) / S);
        mbar_wait(&full[s], (last / S) & 1, nullptr, limit_ns, kSiteDrain);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_i8(kQRows, kQBN);
      // ring positions kept as counters: this thread's instruction count
      // bounds the MMA rate
      const uint32_t dlo0 = desc_sw128_lo(smem_u32(sX));
      int s = 0, t = 0;
      uint32_t tph = 0;   // phase parity of afull[t]
      int i = 0;
      bool stop = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs, ++i) {
        const int b = i & 1;
        if (i >= 2 && !mbar_wait_cluster(&accempty[b], ((i >> 1) & 1) ^ 1u, abort_flag, limit_ns, kSiteAcc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + b * kQAccCols;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait_cluster(&afull[t], tph, abort_flag, limit_ns, kSiteMmaExfull)) {
            stop = true;
            break;
          }
          tc_fence_after();
          // the stage's 16 MMAs (K = 32 each) from one asm block: MMA k reads
          // A column 8k of the slot and token box k / 4, bytes 32 (k % 4)
          static_assert(kQBK == 512, "one stage is sixteen MMAs");
          mma_i8_stage16_pair<kQXBoxBytes / 16>(d_tmem, tmem + kQACol + kQASlotCols * t,
                                                dlo0 + s * (kQXStageBytes / 16), kDescSw128Hi, idesc,
                                                ks != 0 ? 1u : 0u);
          tc_commit_pair(&done[s], 3);
          if (++s == S) s = 0;
          if (++t == kQASlots) {
            t = 0;
            tph ^= 1u;
          }
        }
        if (stop) break;
        tc_commit_pair(&accfull[b], 3);
      }
      // no MMA of the pair may be in flight when either CTA frees its TMEM
      tc_commit_pair(drain, 1);
      mbar_wait(drain, 0, nullptr, limit_ns, kSiteDrain);
    }
  } else if (warp < kQFirstEpi) {
    // ---------------- expanders (both CTAs) ----------------
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // 128-byte swizzle of the packed box: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
    static_assert(kQWRowBytes == 128, "the packed box is 128-byte rows");
    const uint32_t wsw = static_cast<uint32_t>(r & 7);
    uint32_t g = 0;
    bool stop = false;
    for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
      for (int ks = 0; ks < nk; ++ks, ++g) {
        if (static_cast<int>(g % kQExpGroups) != grp) continue;
        const int s = g % S;
        const int t = g % kQASlots;
        bool ok = mbar_wait(&full[s], (g / S) & 1, abort_flag, limit_ns, kSiteExpFull);
        if (ok && g >= static_cast<uint32_t>(kQASlots)) {
          // slot t was last used by stage g - kQASlots: free once that stage is done
          const uint32_t gp = g - kQASlots;
          ok = mbar_wait_cluster(&done[gp % S], (gp / S) & 1, abort_flag, limit_ns, kSiteExpEmpty);
        }
        if (!__all_sync(0xffffffffu, ok)) {
          stop = true;
          break;
        }
        tc_fence_after();
        // row r of the stage: kQWRowBytes packed bytes in 16-byte chunks, 32
        // bytes (K = 128) per tcgen05.st of 32 columns
        const uint32_t wrow = smem_u32(sW + s * kQWStageBytes) + r * kQWRowBytes;
#pragma unroll
        for (int h = 0; h < kQWRowBytes / 32; ++h) {
          const uint4 lo = ld_shared_v4(wrow + (((2u * h) ^ wsw) << 4));
          const uint4 hi = ld_shared_v4(wrow + (((2u * h + 1u) ^ wsw) << 4));
          const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          uint32_t v[32];
#pragma unroll
          for (int gw = 0; gw < 8; ++gw)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[4 * gw + j] = (wd[gw] >> (2 * j)) & 0x03030303u;
          tmem_st_32x32b_x32(tmem + lane_base + kQACol + kQASlotCols * t + 32 * h, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(&afull[t], 0);
      }
    }
  } else {
    // ---------------- epilogue (both CTAs) ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int et = threadIdx.x - 32 * kQFirstEpi;
    const int col0 = ((warp - kQFirstEpi) >> 2) * kQEpiCols;   // this warp's half of the tokens
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float gamma0 = (out_mode == kOutI32) ? 1.f : *P.p[0].gamma;
    const float gamma1 = (out_mode == kOutI32 || P.count < 2) ? 1.f : *P.p[1].gamma;
    int i = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++i) {
      const int b = i & 1;
      const int m0 = (tile % mt) * kQBN;
      const int nt = tile / mt, w = nt >= ntn0 ? 1 : 0;
      const int n0 = (nt - (w ? ntn0 : 0)) * kQRows + static_cast<int>(rank) * kTcRows;
      const QOut& O = P.p[w];
      const int N = O.N;
      void* __restrict__ Y = O.Y;
      const float* __restrict__ bias = O.bias;
      const float gamma = w ? gamma1 : gamma0;
      for (int j = et; j < kQBN; j += 32 * kQEpiWarps) {
        const int m = m0 + j;
        int rv = 0;
        float fv = 0.f;
        if (m < M) {
          rv = Rg[m];
          if (out_mode != kOutI32) fv = __fdiv_rn(gamma, sg[m]);
        }
        sR[b * kQBN + j] = rv;
        sF[b * kQBN + j] = fv;
      }
      __syncwarp();
      named_bar_sync(2, 32 * kQEpiWarps);
      const bool ok = mbar_wait_cluster(&accfull[b], (i >> 1) & 1, abort_flag, limit_ns, kSiteAcc) && !*abort_flag;
      __syncwarp();
      if (!named_bar_and(3, 32 * kQEpiWarps, ok)) break;
      tc_fence_after();
      const int n = n0 + r;
      const float bias_n = (bias && n < N) ? __ldg(bias + n) : 0.f;
      if (O.tma_store) {
        // bf16 tile of this warp, [BN tokens][32 rows], then one TMA store
        uint16_t* so = reinterpret_cast<uint16_t*>(sOut + (warp - kQFirstEpi) * kQStageOutBytes);
        if (lane == 0) bulk_wait_group_read0();   // the previous store has read the buffer
        __syncwarp();
#pragma unroll 1
        for (int c0 = col0; c0 < col0 + kQEpiCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + lane_base + b * kQAccCols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int a = static_cast<int>(v[t]) - sR[b * kQBN + c0 + t];
            float y = __fmul_rn(__int2float_rn(a), sF[b * kQBN + c0 + t]);
            if (bias) y = __fadd_rn(y, bias_n);
            so[(c0 - col0 + t) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
          }
        }
        tc_fence_before();
        mbar_arrive_cluster(&accempty[b], 0);   // accumulator drained: the MMAs may reuse it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && m0 + col0 < M) {   // (a box starting past the last token writes nothing)
          tma_store_2d(&O.tmY, n0 + q * 32, m0 + col0, so);
          bulk_commit_group();
        }
        __syncwarp();
        named_bar_sync(2, 32 * kQEpiWarps);
        continue;
      }
#pragma unroll 1
      for (int c0 = col0; c0 < col0 + kQEpiCols; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + b * kQAccCols + c0, v);
        tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int m = m0 + c0 + t;
            if (m < M) {
              const int a = static_cast<int>(v[t]) - sR[b * kQBN + c0 + t];
              const size_t o = static_cast<size_t>(m) * N + n;
              if (out_mode == kOutI32) {
                static_cast<int*>(Y)[o] = a;
              } else {
                float y = __fmul_rn(__int2float_rn(a), sF[b * kQBN + c0 + t]);
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
      mbar_arrive_cluster(&accempty[b], 0);
      __syncwarp();
      named_bar_sync(2, 32 * kQEpiWarps);
    }
  }
  if (warp >= kQFirstEpi && lane == 0) bulk_wait_group0();   // outputs written before exit
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();   // the leader has drained its MMAs; both CTAs may free TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kQTmemCols);
  }
}

}  // namespace bl
