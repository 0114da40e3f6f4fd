// libbitlinear: host side of the C ABI declared in include/bitlinear.h.
//
// Validation happens before any CUDA call, so a rejected call launches
// nothing (and needs no GPU).  Dispatch:
//   M <= 2      decode GEMV with the activation quantisation fused in;
//   otherwise   activation quantisation into the caller's workspace, then the
//               tcgen05 kind::i8 GEMM (weights expanded into tensor memory).
#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/bitlinear.h"
#include "bl_act.cuh"
#include "bl_common.cuh"
#include "bl_copy.cuh"
#include "bl_tc_common.cuh"
#include "bl_gemm_tc2.cuh"
#include "bl_gemm_2sm.cuh"
#include "bl_gemv.cuh"
#include "bl_decode.cuh"
#include "bl_probe.cuh"
#include "bl_weights.cuh"

namespace {

constexpr int kVersion = 100;                       // 0.1.0
constexpr int64_t kMaxK = 65536;
constexpr int64_t kMaxElems = int64_t(1) << 40;     // N*K and M*K bound
constexpr int kGemvMaxM = 2;
constexpr int kAbsumMaxBlocks = 592;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr int kMaxDevices = 64;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// An NVTX range around each public call (visible in Nsight timelines; a
// no-op unless a profiling tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bl_status check_shape_nk(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || (K % 64) != 0 || K > kMaxK) return BL_ERR_SHAPE;
  if (N >= kMaxElems / K) return BL_ERR_SHAPE;
  return BL_OK;
}

bl_status check_m(int64_t M, int64_t K) {
  if (M < 0 || M > INT32_MAX) return BL_ERR_SHAPE;
  if (M > 0 && M >= kMaxElems / K) return BL_ERR_SHAPE;
  return BL_OK;
}

bl_status last_cuda() { return cudaGetLastError() == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Raise a kernel's dynamic shared memory limit once per device.
template <typename F>
bool ensure_smem(F* func, int bytes, std::atomic<uint64_t>* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  const uint64_t bit = uint64_t(1) << dev;
  if (done_mask->load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(func), cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done_mask->fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || p == nullptr)
    return nullptr;
  f = reinterpret_cast<EncodeTiledFn>(p);
  fn.store(f, std::memory_order_release);
  return f;
}

// 2-D uint8 tensor [rows, cols] (cols contiguous), box [box_rows, box_cols].
bool encode_u8_2d(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                  uint32_t box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// launches
// ---------------------------------------------------------------------------

template <int MT, int RT>
bl_status launch_gemv_t(const void* X, int x_is_i8, int M, int K, int N, const uint8_t* Wp, const float* gamma, int Q,
                        void* Y, int out_mode, cudaStream_t stream) {
  static std::atomic<uint64_t> done{0};
  const int KL = static_cast<int>(align_up(static_cast<size_t>(K), 128));
  const int smem = MT * KL;
  if (!ensure_smem(bl::bl_decode_long_kernel<MT, RT>, MT * static_cast<int>(kMaxK), &done)) return BL_ERR_CUDA;
  const int ntiles = (N + RT - 1) / RT;
  int blocks = (ntiles + bl::kGemvWarps - 1) / bl::kGemvWarps;
  const int cap = 2 * num_sms();
  if (blocks > cap) blocks = cap;
  bl::bl_decode_long_kernel<MT, RT><<<blocks, bl::kGemvThreads, smem, stream>>>(
      X, x_is_i8, M, K, N, reinterpret_cast<const uint4*>(Wp), gamma, Q, Y, out_mode);
  return last_cuda();
}

template <int MT, int CPL, int RT, int D, int THREADS, int MINB>
bl_status launch_gemv1_t(const void* X, int x_is_i8, int K, int N, const uint8_t* Wp, const float* gamma, int Q,
                         void* Y, int out_mode, cudaStream_t stream) {
  constexpr int kWarps = THREADS / 32;
  const int ntiles = (N + RT - 1) / RT;
  // spread the tiles over at most MINB CTAs per SM, every CTA a contiguous range
  const int cap = MINB * num_sms();
  int tiles_per_cta = (ntiles + cap - 1) / cap;
  if (tiles_per_cta < kWarps) tiles_per_cta = (ntiles < kWarps) ? ntiles : kWarps;
  const int blocks = (ntiles + tiles_per_cta - 1) / tiles_per_cta;
  // programmatic dependent launch: the kernel only prefetches into L2 before
  // its griddepcontrol.wait, so it may start while the previous kernel drains
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint4* wp4 = reinterpret_cast<const uint4*>(Wp);
  if (cudaLaunchKernelEx(&cfg, bl::bl_decode_rows_kernel<MT, CPL, RT, D, THREADS, MINB>, X, x_is_i8, K, N, wp4, gamma, Q, Y,
                         out_mode, tiles_per_cta) != cudaSuccess)
    return BL_ERR_CUDA;
  return last_cuda();
}

// ---------------------------------------------------------------------------
// One-token problems: the decode kernel (bl_decode_kernel), resident or big
// ring mode.
// ---------------------------------------------------------------------------

template <int A, int PRE, int FMT, int MODE>
bl_status launch_dec_t(const bl::G2Table& tab, int grid, int in_mode, int Q, int out_mode, cudaStream_t stream) {
  auto kern = bl::bl_decode_kernel<A, PRE, FMT, MODE>;
  constexpr int smem = bl::dec_smem_bytes(MODE, FMT);
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
  if (!(done.load(std::memory_order_acquire) & (uint64_t(1) << dev))) {
    // two CTAs per SM (this launch's and the next one's) need the largest
    // shared-memory carve-out; big mode with base-3 rows: one CTA takes most of it
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess ||
        cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return BL_ERR_CUDA;
    done.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(bl::dec_threads(MODE, FMT));
  // the same footprint for every launch: a third CTA never fits on an SM, so
  // two CTAs of one launch never share an SM
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const unsigned long long lim = kWaitLimitNs;
  if (cudaLaunchKernelEx(&cfg, kern, tab, in_mode, Q, out_mode, lim) != cudaSuccess) return BL_ERR_CUDA;
  return last_cuda();
}

template <int PRE>
bl_status launch_dec_resident(int wplr, const bl::G2Table& tab, int grid, int in_mode, int Q, int out_mode,
                              cudaStream_t stream) {
  constexpr int F = bl::kFmt2Bit, M = bl::kModeResident;
  switch (wplr) {
    case 1: return launch_dec_t<1, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    case 2: return launch_dec_t<2, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    case 3: return launch_dec_t<3, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    case 4: return launch_dec_t<4, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    default: return launch_dec_t<5, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
  }
}

template <int PRE>
bl_status launch_dec_big(int cpl, const bl::G2Table& tab, int grid, int in_mode, int Q, int out_mode,
                         cudaStream_t stream) {
  constexpr int F = bl::kFmt2Bit, M = bl::kModeBig;
  switch (cpl) {
    case 1: return launch_dec_t<1, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    case 2: return launch_dec_t<2, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    case 3: return launch_dec_t<3, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
    default: return launch_dec_t<4, PRE, F, M>(tab, grid, in_mode, Q, out_mode, stream);
  }
}

// Words of 16 weights per lane for a row of K weights (resident mode).
inline int dec_wpl(int64_t K) { return static_cast<int>((K + 511) / 512); }
// 16-byte chunks per lane (big mode).
inline int dec_cpl(int64_t K) { return static_cast<int>((K + 2047) / 2048); }

// The register width A of one resident launch (words of codes a lane keeps,
// <= 5): the words-per-lane class that holds the most weight bytes (5 if no
// problem has K <= 2560), raised so that no row needs more than
// kDecMaxSplit warps.  Longer rows are split across a team of warps.
int dec_pick_wplr(const bl_linear* const* probs, int n) {
  double bytes[bl::kDecRegMaxWpl + 1] = {};
  int64_t max_words = 0;
  for (int i = 0; i < n; ++i) {
    const int w = dec_wpl(probs[i]->K);
    if (w <= bl::kDecRegMaxWpl) bytes[w] += static_cast<double>(probs[i]->N) * static_cast<double>(probs[i]->K);
    max_words = std::max<int64_t>(max_words, probs[i]->K / 16);
  }
  int best = bl::kDecRegMaxWpl;
  double most = 0.0;
  for (int w = 1; w <= bl::kDecRegMaxWpl; ++w)
    if (bytes[w] > most) {
      most = bytes[w];
      best = w;
    }
  const int floor_a = static_cast<int>((max_words + 32 * bl::kDecMaxSplit - 1) / (32 * bl::kDecMaxSplit));
  return std::max(best, floor_a);
}

// Warps that split one row of K weights at register width a (resident 2-bit).
inline int dec_split(int64_t K, int a) { return static_cast<int>((K / 16 + 32 * a - 1) / (32 * a)); }

// Bytes of one stored row.
inline int dec_row_bytes(int64_t K, int fmt) {
  return fmt == bl::kFmtBase3 ? 4 * bl::base3_row_words(static_cast<int>(K)) : static_cast<int>(K / 4);
}

// Rows a warp (team) takes at once.
inline int dec_rt(int mode, int fmt) {
  if (mode == bl::kModeBig) return bl::kDecBigRows;
  return fmt == bl::kFmt2Bit ? bl::kDecRegRows : bl::kDecB3Rows;
}

// Estimated time of one CTA of a problem that gets `ctas` CTAs.  Resident
// mode: rounds of row groups over the CTA's teams of warps times the cost of
// a group (issue slots of one warp: per word a lane keeps, two shared loads,
// eight masks and eight dp4a at half rate for the two rows; the rows'
// reductions and stores; shared adds when rows are split), plus a penalty
// for bytes that do not fit the ring (fetched after the dependency wait).
// Big mode: the weight bytes a CTA streams.
// Row-lane mode: issue slots of one SM sub-partition (items go round-robin
// to 16 warps, four per sub-partition): per 16-byte column of a 32-row tile
// about 37 instructions, per item (tile x 512-weight segment) about 25 more;
// bytes beyond the ring as above; more than 512 rows a CTA is not allowed.
double dec_cta_cost(int64_t N, int64_t K, int ctas, int a, int fmt, int mode) {
  const int64_t rows = (N + ctas - 1) / ctas;
  const double bytes = static_cast<double>(rows) * static_cast<double>(dec_row_bytes(K, fmt));
  if (mode == bl::kModeBig) return bytes;
  if (mode == bl::kModeRowLane) {
    if (rows > bl::kDecLaneMaxRows) return 1e12;
    const int64_t tiles = (rows + bl::kDecLaneRows - 1) / bl::kDecLaneRows;
    const int64_t upr = K / 64, segs = (upr + 7) / 8;
    const double pb = static_cast<double>(rows) * bl::dec_lane_stride(static_cast<int>(K / 4));
    const double over = pb > bl::kDecRingBytes ? (pb - bl::kDecRingBytes) / 8.0 : 0.0;
    return (static_cast<double>(tiles * upr) * 37.0 + static_cast<double>(tiles * segs) * 25.0) / 4.0 + over;
  }
  const int rt = dec_rt(mode, fmt);
  const int64_t groups = (rows + rt - 1) / rt;
  double group;
  int teams;
  if (fmt == bl::kFmtBase3) {
    group = ((bl::base3_row_words(static_cast<int>(K)) + 31) / 32) * 140.0 + 70.0;
    teams = bl::kDecWarps;
  } else {
    const int S = dec_split(K, a);
    group = a * 26.0 + 40.0 + (S > 1 ? 10.0 : 0.0);
    teams = bl::kDecWarps / S;
  }
  const int64_t rounds = (groups + teams - 1) / teams;
  const double over = bytes > bl::kDecRingBytes ? (bytes - bl::kDecRingBytes) / 8.0 : 0.0;
  return static_cast<double>(rounds) * group + over;
}

// Fill a launch table with one-token problems: CTAs are shared out so that
// the slowest CTA (by the cost model above) is as fast as possible, and the
// launch has exactly one CTA per SM when the rows allow.  Each problem's row
// range per CTA is cut into whole-group chunks: in resident mode as few as
// fit the ring without reuse when possible; in big mode one group per warp
// per chunk.  Returns the grid size.
void plan_decode(const bl_linear* const* probs, int n, int sms, int mode, int a, int fmt, int* c, int* crs,
                 int* sls) {
  int64_t rows_total = 0;
  for (int i = 0; i < n; ++i) rows_total += probs[i]->N;
  const int target = static_cast<int>(rows_total < sms ? rows_total : sms);
  // smallest CTA count of problem i whose cost is <= T
  auto need = [&](int i, double T) {
    const int64_t Nn = probs[i]->N;
    int lo = 1, hi = static_cast<int>(Nn < target ? Nn : target);
    if (dec_cta_cost(Nn, probs[i]->K, hi, a, fmt, mode) > T) return hi + 1;   // infeasible
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if (dec_cta_cost(Nn, probs[i]->K, mid, a, fmt, mode) <= T)
        hi = mid;
      else
        lo = mid + 1;
    }
    return lo;
  };
  // the smallest makespan that fits the grid: binary search over the costs
  double lo_t = 0.0, hi_t = 0.0;
  for (int i = 0; i < n; ++i)
    hi_t = std::max(hi_t, dec_cta_cost(probs[i]->N, probs[i]->K, 1, a, fmt, mode));
  for (int it = 0; it < 60; ++it) {
    const double mid = 0.5 * (lo_t + hi_t);
    int sum = 0;
    for (int i = 0; i < n; ++i) sum += need(i, mid);
    if (sum <= target)
      hi_t = mid;
    else
      lo_t = mid;
  }
  int sum = 0;
  for (int i = 0; i < n; ++i) {
    c[i] = need(i, hi_t);
    sum += c[i];
  }
  // spare CTAs go to the problems with the most weight bytes per CTA
  while (sum < target) {
    int best = -1;
    double most = 0.0;
    for (int i = 0; i < n; ++i) {
      if (c[i] >= probs[i]->N) continue;
      const double per = static_cast<double>(probs[i]->N) * static_cast<double>(probs[i]->K) / c[i];
      if (per > most) {
        most = per;
        best = i;
      }
    }
    if (best < 0) break;
    c[best] += 1;
    sum += 1;
  }
  const int ring = bl::dec_ring_bytes(mode, fmt);
  const int chunk_max = bl::dec_chunk_max(mode, fmt);
  for (int i = 0; i < n; ++i) {
    const bl_linear& p = *probs[i];
    const int rb = dec_row_bytes(p.K, fmt);
    const int rt = dec_rt(mode, fmt);
    const int maxrows = static_cast<int>((p.N + c[i] - 1) / c[i]);
    int cr = (chunk_max / rb) / rt * rt, slots = 0;
    if (mode == bl::kModeRowLane) {
      // one 32-row tile a chunk; every chunk resident when the padded rows fit
      const int st = bl::dec_lane_stride(rb);
      cr = bl::kDecLaneRows;
      const int nch = (maxrows + cr - 1) / cr;
      slots = (static_cast<int64_t>(maxrows) * st <= ring) ? nch : ring / (cr * st);
      crs[i] = cr;
      sls[i] = std::max(1, std::min(bl::kDecMaxSlots, slots));
      continue;
    }
    if (mode == bl::kModeResident && fmt == bl::kFmt2Bit && dec_split(p.K, a) > 1)
      cr = std::min(cr, bl::kDecSplitRows / rt * rt);   // split rows: the chunk's totals in shared memory
    if (mode == bl::kModeBig) {
      // one group per consumer warp per chunk
      cr = std::min(cr, bl::dec_warps(mode, fmt) * rt);
      slots = std::min(bl::kDecMaxSlots, ring / (cr * rb));
    } else {
      const int cr_max = cr;
      for (; cr >= rt; cr -= rt) {
        slots = std::min(bl::kDecMaxSlots, ring / (cr * rb));
        if ((maxrows + cr - 1) / cr <= slots) break;
      }
      if (cr < rt) {
        cr = cr_max;
        slots = std::min(bl::kDecMaxSlots, ring / (cr * rb));
      }
    }
    crs[i] = cr;
    sls[i] = slots;
  }
}

// The shape-only part of a launch table (CTAs per problem, chunk rows,
// slots) depends on the problems' N and K, the mode, the register width and
// the SM count alone; the search above costs more host time than the launch,
// so recent plans are kept (a small round-robin table).
struct DecPlan {
  int n = 0, sms = 0, mode = 0, a = 0, fmt = 0;
  int64_t N[bl::kG2MaxProblems] = {}, K[bl::kG2MaxProblems] = {};
  int c[bl::kG2MaxProblems] = {}, cr[bl::kG2MaxProblems] = {}, slots[bl::kG2MaxProblems] = {};
};
constexpr int kDecPlanCache = 16;

void plan_decode_cached(const bl_linear* const* probs, int n, int sms, int mode, int a, int fmt, int* c, int* crs,
                        int* sls) {
  static std::mutex mu;
  static DecPlan plans[kDecPlanCache];
  static int used = 0, next = 0;
  auto same = [&](const DecPlan& q) {
    if (q.n != n || q.sms != sms || q.mode != mode || q.a != a || q.fmt != fmt) return false;
    for (int i = 0; i < n; ++i)
      if (q.N[i] != probs[i]->N || q.K[i] != probs[i]->K) return false;
    return true;
  };
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int e = 0; e < used; ++e)
      if (same(plans[e])) {
        for (int i = 0; i < n; ++i) {
          c[i] = plans[e].c[i];
          crs[i] = plans[e].cr[i];
          sls[i] = plans[e].slots[i];
        }
        return;
      }
  }
  plan_decode(probs, n, sms, mode, a, fmt, c, crs, sls);
  DecPlan q;
  q.n = n;
  q.sms = sms;
  q.mode = mode;
  q.a = a;
  q.fmt = fmt;
  for (int i = 0; i < n; ++i) {
    q.N[i] = probs[i]->N;
    q.K[i] = probs[i]->K;
    q.c[i] = c[i];
    q.cr[i] = crs[i];
    q.slots[i] = sls[i];
  }
  std::lock_guard<std::mutex> lock(mu);
  plans[next] = q;
  next = (next + 1) % kDecPlanCache;
  if (used < kDecPlanCache) ++used;
}

int fill_decode_table(bl::G2Table* tab, const bl_linear* const* probs, int n, int sms, int mode, int a,
                      const void* const* Us, const float* bias, float eps, int fmt = bl::kFmt2Bit) {
  std::memset(tab, 0, sizeof(*tab));
  int c[bl::kG2MaxProblems], crs[bl::kG2MaxProblems], sls[bl::kG2MaxProblems];
  plan_decode_cached(probs, n, sms, mode, a, fmt, c, crs, sls);
  int grid = 0;
  for (int i = 0; i < n; ++i) {
    const bl_linear& p = *probs[i];
    bl::G2Problem& q = tab->p[i];
    q.X = p.X;
    q.U = Us ? Us[i] : nullptr;
    q.Wp = p.Wp;
    q.gamma = p.gamma;
    q.Y = p.Y;
    q.K = static_cast<int>(p.K);
    q.N = static_cast<int>(p.N);
    q.rows_per_cta = static_cast<int>(p.N / c[i]);
    q.rows_rem = static_cast<int>(p.N % c[i]);
    q.cta_begin = grid;
    q.ctas = c[i];
    q.bias = bias;
    q.eps = eps;
    q.chunk_rows = crs[i];
    q.slots = sls[i];
    q.ksplit = (mode == bl::kModeResident && fmt == bl::kFmt2Bit) ? dec_split(p.K, a) : 1;
    grid += c[i];
  }
  tab->count = n;
  return grid;
}

// Launch one-token problems (K <= 8192, at most kG2MaxProblems) in one kernel:
// resident mode when the weights fit the rings of one CTA per SM, big mode
// otherwise (the normalising prologues exist only in resident mode; callers
// check the fit).  in_mode: bl::InMode of the token input; Us: per problem,
// the up projection's output in the gated squared-ReLU mode or the RMSNorm
// weight (NULL array: none); eps: the normalisation epsilon.
bl_status launch_decode(const bl_linear* const* probs, int n, int in_mode, int Q, int out_mode, cudaStream_t stream,
                        const void* const* Us = nullptr, const float* bias = nullptr, float eps = 0.f) {
  if (n <= 0) return BL_OK;
  const int sms = num_sms();
  double wbytes = 0.0;
  int maxK = 64;
  for (int i = 0; i < n; ++i) {
    wbytes += static_cast<double>(probs[i]->N) * static_cast<double>(probs[i]->K) / 4.0;
    if (probs[i]->K > maxK) maxK = static_cast<int>(probs[i]->K);
  }
  const bool norm = in_mode == bl::kInRmsNorm || in_mode == bl::kInLayerNorm;
  const bool big = !norm && wbytes > static_cast<double>(sms) * bl::kDecRingBytes;
  const bool relu2 = in_mode == bl::kInRelu2 || in_mode == bl::kInRelu2Gated;
  bl::G2Table tab;
  if (!big) {
    // row-lane mode when every CTA's rows fit its shared row totals
    const int grid = fill_decode_table(&tab, probs, n, sms, bl::kModeRowLane, 0, Us, bias, eps);
    bool fits = true;
    for (int i = 0; i < n; ++i)
      fits = fits && tab.p[i].rows_per_cta + (tab.p[i].rows_rem ? 1 : 0) <= bl::kDecLaneMaxRows;
    if (fits) {
      if (relu2) return launch_dec_t<0, bl::kDecRelu2, bl::kFmt2Bit, bl::kModeRowLane>(tab, grid, in_mode, Q, out_mode, stream);
      if (in_mode == bl::kInRmsNorm)
        return launch_dec_t<0, bl::kDecRms, bl::kFmt2Bit, bl::kModeRowLane>(tab, grid, in_mode, Q, out_mode, stream);
      if (in_mode == bl::kInLayerNorm)
        return launch_dec_t<0, bl::kDecLn, bl::kFmt2Bit, bl::kModeRowLane>(tab, grid, in_mode, Q, out_mode, stream);
      return launch_dec_t<0, bl::kDecPlain, bl::kFmt2Bit, bl::kModeRowLane>(tab, grid, in_mode, Q, out_mode, stream);
    }
  }
  const int mode = big ? bl::kModeBig : bl::kModeResident;
  const int a = big ? dec_cpl(maxK) : dec_pick_wplr(probs, n);
  const int grid = fill_decode_table(&tab, probs, n, sms, mode, a, Us, bias, eps);
  if (big) {
    if (relu2) return launch_dec_big<bl::kDecRelu2>(a, tab, grid, in_mode, Q, out_mode, stream);
    return launch_dec_big<bl::kDecPlain>(a, tab, grid, in_mode, Q, out_mode, stream);
  }
  if (relu2) return launch_dec_resident<bl::kDecRelu2>(a, tab, grid, in_mode, Q, out_mode, stream);
  if (in_mode == bl::kInRmsNorm) return launch_dec_resident<bl::kDecRms>(a, tab, grid, in_mode, Q, out_mode, stream);
  if (in_mode == bl::kInLayerNorm) return launch_dec_resident<bl::kDecLn>(a, tab, grid, in_mode, Q, out_mode, stream);
  return launch_dec_resident<bl::kDecPlain>(a, tab, grid, in_mode, Q, out_mode, stream);
}

// Single one-token problem.
bl_status launch_decode_one(const void* X, int x_is_i8, int K, int N, const uint8_t* Wp, const float* gamma, int Q,
                            void* Y, int out_mode, cudaStream_t stream) {
  bl_linear p;
  p.X = static_cast<const uint16_t*>(X);
  p.M = 1;
  p.K = K;
  p.N = N;
  p.Wp = Wp;
  p.gamma = gamma;
  p.Y = static_cast<uint16_t*>(Y);
  const bl_linear* pp = &p;
  return launch_decode(&pp, 1, x_is_i8, Q, out_mode, stream);
}

// One token with K <= 8192: the decode kernels; two tokens: the register-ring
// GEMV; longer rows: the general GEMV.
bl_status launch_gemv(const void* X, int x_is_i8, int M, int K, int N, const uint8_t* Wp, const float* gamma, int Q,
                      void* Y, int out_mode, cudaStream_t stream) {
  if (M == 1 && K <= bl::kDecMaxK) return launch_decode_one(X, x_is_i8, K, N, Wp, gamma, Q, Y, out_mode, stream);
  const int cpl = (K / 64 + 31) / 32;
  // one CTA of 16 warps per SM (room for the next kernel's CTA to start its
  // L2 prefetch alongside); D tiles of weights in flight per warp
  if (M == 2 && K <= 4096) {
    if (cpl == 1) return launch_gemv1_t<2, 1, 2, 2, 512, 1>(X, x_is_i8, K, N, Wp, gamma, Q, Y, out_mode, stream);
    return launch_gemv1_t<2, 2, 1, 2, 512, 1>(X, x_is_i8, K, N, Wp, gamma, Q, Y, out_mode, stream);
  }
  if (M == 1) return launch_gemv_t<1, 2>(X, x_is_i8, M, K, N, Wp, gamma, Q, Y, out_mode, stream);
  return launch_gemv_t<2, 2>(X, x_is_i8, M, K, N, Wp, gamma, Q, Y, out_mode, stream);
}

// Per-token activation quantisation: a warp per row when there are rows enough
// to fill the GPU and a row fits a warp's registers, a CTA per row otherwise.
bl_status launch_act_quant(const uint16_t* X, int m, int k, int Q, int8_t* Xq, float* s, int* R, cudaStream_t stream) {
  // measured: the CTA-per-row kernel also wins for long rows (K > 4096, where
  // a warp can no longer keep its row in registers and reads part of it twice)
  if (m < bl::kActRowsPerBlock * num_sms() || k > 32 * 8 * bl::kActCache) {
    bl::bl_act_quant_row_kernel<false><<<m, bl::kActRowThreads, 0, stream>>>(X, k, Q, Xq, s, R, nullptr);
  } else {
    const int blocks = (m + bl::kActRowsPerBlock - 1) / bl::kActRowsPerBlock;
    bl::bl_act_quant_kernel<<<blocks, 256, 0, stream>>>(X, m, k, Q, Xq, s, R);
  }
  return last_cuda();
}

template <int BN, int EXPG>
bl_status launch_tc2_t(const int8_t* Xq, int M, int K, int N, const uint8_t* Wp, const int* R, const float* s,
                       const float* gamma, void* Y, int out_mode, cudaStream_t stream, const float* bias) {
  using C = bl::P2Cfg<BN>;
  static std::atomic<uint64_t> done{0};
  if (!ensure_smem(bl::bl_mma_persistent_kernel<BN, EXPG>, C::kSmemBytes, &done)) return BL_ERR_CUDA;
  CUtensorMap tmX, tmW;
  if (!encode_u8_2d(&tmX, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K), BN, bl::kTcBK,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BL_ERR_CUDA;
  if (!encode_u8_2d(&tmW, Wp, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4), bl::kTcRows, bl::kP2BK / 4,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BL_ERR_CUDA;
  const int ntiles = ((M + BN - 1) / BN) * ((N + bl::kTcRows - 1) / bl::kTcRows);
  const int grid = ntiles < num_sms() ? ntiles : num_sms();
  bl::bl_mma_persistent_kernel<BN, EXPG><<<grid, bl::P2Warps<EXPG>::kThreads, C::kSmemBytes, stream>>>(
      tmX, tmW, M, N, K, R, s, gamma, Y, out_mode, bias, kWaitLimitNs);
  return last_cuda();
}

// Largest number of two-CTA clusters of `kernel` that are resident at once on
// the current device (cached per device).
template <typename F>
int max_active_pairs(F* kernel, int threads, int smem) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) return 0;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// One weight tensor of a tensor-core launch.
struct TcProb {
  const uint8_t* Wp;
  const float* gamma;
  void* Y;
  int N;
  const float* bias;
};

// The CTA-pair GEMM over one or two problems that share the quantised
// activations Xq [M, K] (its tiles run over both weight tensors).
bl_status launch_tc_pair_multi(const int8_t* Xq, int M, int K, const TcProb* probs, int count, const int* R,
                               const float* s, int out_mode, cudaStream_t stream) {
  static std::atomic<uint64_t> done{0};
  if (!ensure_smem(bl::bl_mma_pair_kernel, bl::kQSmemBytes, &done)) return BL_ERR_CUDA;
  CUtensorMap tmX;
  if (!encode_u8_2d(&tmX, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K), bl::kQHalf, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BL_ERR_CUDA;
  bl::QProblems P;
  std::memset(&P, 0, sizeof(P));
  P.count = count;
  int ntn = 0;
  for (int w = 0; w < count; ++w) {
    const TcProb& q = probs[w];
    bl::QOut& O = P.p[w];
    if (!encode_u8_2d(&O.tmW, q.Wp, static_cast<uint64_t>(q.N), static_cast<uint64_t>(K / 4), bl::kTcRows,
                      bl::kQBK / 4, CU_TENSOR_MAP_SWIZZLE_128B))
      return BL_ERR_CUDA;
    // bf16 outputs leave through TMA stores when the rows are 16-byte aligned
    if (out_mode == bl::kOutBF16 && (q.N % 8) == 0 && (reinterpret_cast<uintptr_t>(q.Y) & 15u) == 0) {
      EncodeTiledFn enc = get_encode();
      if (!enc) return BL_ERR_CUDA;
      const cuuint64_t dims[2] = {static_cast<cuuint64_t>(q.N), static_cast<cuuint64_t>(M)};
      const cuuint64_t strides[1] = {static_cast<cuuint64_t>(q.N) * 2};
      const cuuint32_t box[2] = {32, static_cast<cuuint32_t>(bl::kQEpiCols)};
      const cuuint32_t estr[2] = {1, 1};
      if (enc(&O.tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.Y, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return BL_ERR_CUDA;
      O.tma_store = 1;
    }
    O.gamma = q.gamma;
    O.Y = q.Y;
    O.bias = q.bias;
    O.N = q.N;
    O.ntn = (q.N + bl::kQRows - 1) / bl::kQRows;
    ntn += O.ntn;
  }
  const int ntiles = ((M + bl::kQBN - 1) / bl::kQBN) * ntn;
  cudaLaunchConfig_t cfg = {};
  // a persistent grid must fit in one wave: not every SM can host half of a
  // two-SM cluster, so ask how many clusters are co-resident (once per device)
  int npairs = max_active_pairs(bl::bl_mma_pair_kernel, bl::kQThreads, bl::kQSmemBytes);
  if (npairs <= 0) return BL_ERR_CUDA;
  if (npairs > ntiles) npairs = ntiles;
  cfg.gridDim = dim3(2 * npairs);
  cfg.blockDim = dim3(bl::kQThreads);
  cfg.dynamicSmemBytes = bl::kQSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const unsigned long long lim = kWaitLimitNs;
  if (cudaLaunchKernelEx(&cfg, bl::bl_mma_pair_kernel, tmX, P, M, K, R, s, out_mode, lim) != cudaSuccess)
    return BL_ERR_CUDA;
  return last_cuda();
}

bl_status launch_tc_pair(const int8_t* Xq, int M, int K, int N, const uint8_t* Wp, const int* R, const float* s,
                         const float* gamma, void* Y, int out_mode, cudaStream_t stream, const float* bias) {
  const TcProb p{Wp, gamma, Y, N, bias};
  return launch_tc_pair_multi(Xq, M, K, &p, 1, R, s, out_mode, stream);
}

// Tensor-core GEMM by token count: the CTA-pair kernel for M > 64, the
// one-SM persistent kernel (token tile 16, 32 or 64) otherwise.
bl_status launch_tc(const int8_t* Xq, int M, int K, int N, const uint8_t* Wp, const int* R, const float* s,
                    const float* gamma, void* Y, int out_mode, cudaStream_t stream, const float* bias = nullptr) {
  if (M > 64) return launch_tc_pair(Xq, M, K, N, Wp, R, s, gamma, Y, out_mode, stream, bias);
  if (M <= 16) return launch_tc2_t<16, 1>(Xq, M, K, N, Wp, R, s, gamma, Y, out_mode, stream, bias);
  if (M <= 32) return launch_tc2_t<32, 1>(Xq, M, K, N, Wp, R, s, gamma, Y, out_mode, stream, bias);
  return launch_tc2_t<64, 1>(Xq, M, K, N, Wp, R, s, gamma, Y, out_mode, stream, bias);
}

struct FwdWs {
  int8_t* Xq;
  float* s;
  int* R;
};

size_t fwd_ws_bytes(int64_t M, int64_t K) {
  if (M <= kGemvMaxM) return 0;
  return align_up(static_cast<size_t>(M) * K, 256) + 2 * align_up(static_cast<size_t>(M) * 4, 256);
}

FwdWs fwd_ws_split(void* ws, int64_t M, int64_t K) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  FwdWs w;
  w.Xq = reinterpret_cast<int8_t*>(p);
  p += align_up(static_cast<size_t>(M) * K, 256);
  w.s = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(M) * 4, 256);
  w.R = reinterpret_cast<int*>(p);
  return w;
}

bl_status forward_common(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                         int bits, void* Y, int out_mode, void* ws, size_t ws_bytes, cudaStream_t stream) {
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!X || !Wp || !gamma || !Y) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wp)) return BL_ERR_ALIGNMENT;
  const size_t need = fwd_ws_bytes(M, K);
  if (need > 0) {
    if (!ws || ws_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(ws)) return BL_ERR_ALIGNMENT;
  }
  const int Q = bits == 8 ? 127 : 7;
  const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
  if (M <= kGemvMaxM) return launch_gemv(X, 0, m, k, n, Wp, gamma, Q, Y, out_mode, stream);
  const FwdWs w = fwd_ws_split(ws, M, K);
  if ((st = launch_act_quant(X, m, k, Q, w.Xq, w.s, w.R, stream)) != BL_OK) return st;
  return launch_tc(w.Xq, m, k, n, Wp, w.R, w.s, gamma, Y, out_mode, stream);
}

}  // namespace

extern "C" {

const char* bl_status_string(bl_status s) {
  switch (s) {
    case BL_OK: return "ok";
    case BL_ERR_INVALID_ARG: return "invalid argument (null pointer)";
    case BL_ERR_SHAPE: return "unsupported shape (need N,K > 0, K % 64 == 0, K <= 65536, M >= 0, N*K < 2^40)";
    case BL_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case BL_ERR_UNSUPPORTED: return "unsupported activation width (bits must be 4 or 8)";
    case BL_ERR_CUDA: return "CUDA error";
    case BL_ERR_TIMEOUT: return "a kernel wait timed out";
    case BL_ERR_WORKSPACE: return "workspace missing or too small";
    case BL_ERR_SCRATCH_LIMIT:
      return "shape exceeds the built-in scratch of bl_forward_noalloc (M*K <= 16 MiB, M <= 8192)";
  }
  return "unknown status";
}

int bl_version(void) { return kVersion; }

size_t bl_packed_weight_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) / 4;
}

static int absum_blocks(int64_t N, int64_t K) {
  const int64_t n4 = N * K / 4;
  int64_t b = (n4 + 255) / 256;
  if (b > kAbsumMaxBlocks) b = kAbsumMaxBlocks;
  if (b < 1) b = 1;
  return static_cast<int>(b);
}

size_t bl_quantize_weights_workspace_bytes(int64_t N, int64_t K) {
  if (check_shape_nk(N, K) != BL_OK) return 0;
  return static_cast<size_t>(bl::kAbsumTotals) * sizeof(unsigned long long);
}

bl_status bl_quantize_weights(const float* W, int64_t N, int64_t K, uint8_t* Wp, float* gamma, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quantize_weights");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if (!W || !Wp || !gamma) return BL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wp)) return BL_ERR_ALIGNMENT;
  const size_t need = bl_quantize_weights_workspace_bytes(N, K);
  if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  const int blocks = absum_blocks(N, K);
  auto* bins = static_cast<unsigned long long*>(workspace);
  const int64_t n = N * K;
  if (cudaMemsetAsync(bins, 0, bl::kAbsumTotals * sizeof(unsigned long long), stream) != cudaSuccess)
    return BL_ERR_CUDA;
  bl::bl_weight_absum_kernel<<<blocks, bl::kAbsumThreads, 0, stream>>>(W, n, bins);
  if ((st = last_cuda()) != BL_OK) return st;
  bl::bl_weight_gamma_kernel<<<1, 32, 0, stream>>>(bins, static_cast<uint64_t>(n), gamma);
  if ((st = last_cuda()) != BL_OK) return st;
  const int64_t nwords = n / 16;
  bl::bl_weight_pack_kernel<<<static_cast<unsigned>((nwords + 255) / 256), 256, 0, stream>>>(
      W, nwords, gamma, reinterpret_cast<uint32_t*>(Wp));
  return last_cuda();
}

bl_status bl_unpack_weights(const uint8_t* Wp, int64_t N, int64_t K, int8_t* codes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_unpack_weights");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if (!Wp || !codes) return BL_ERR_INVALID_ARG;
  if (!aligned16(Wp) || !aligned16(codes)) return BL_ERR_ALIGNMENT;
  const int64_t nwords = N * K / 16;
  bl::bl_weight_unpack_kernel<<<static_cast<unsigned>((nwords + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(Wp), nwords, codes);
  return last_cuda();
}

bl_status bl_quant_act(const uint16_t* X, int64_t M, int64_t K, int bits, int8_t* Xq, float* scale,
                       cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quant_act");
  if (K <= 0 || (K % 64) != 0 || K > kMaxK) return BL_ERR_SHAPE;
  bl_status st = check_m(M, K);
  if (st != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!X || !Xq || !scale) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq)) return BL_ERR_ALIGNMENT;
  return launch_act_quant(X, static_cast<int>(M), static_cast<int>(K), bits == 8 ? 127 : 7, Xq, scale, nullptr,
                          stream);
}

bl_status bl_quant_act_packed4(const uint16_t* X, int64_t M, int64_t K, uint8_t* Xq4, float* scale,
                               cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quant_act_packed4");
  if (K <= 0 || (K % 64) != 0 || K > kMaxK) return BL_ERR_SHAPE;
  bl_status st = check_m(M, K);
  if (st != BL_OK) return st;
  if (M == 0) return BL_OK;
  if (!X || !Xq4 || !scale) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq4)) return BL_ERR_ALIGNMENT;
  bl::bl_act_quant_row_kernel<true><<<static_cast<unsigned>(M), bl::kActRowThreads, 0, stream>>>(
      X, static_cast<int>(K), 7, reinterpret_cast<int8_t*>(Xq4), scale, nullptr, nullptr);
  return last_cuda();
}

size_t bl_forward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  (void)bits;
  if (check_shape_nk(N, K) != BL_OK || check_m(M, K) != BL_OK) return 0;
  return fwd_ws_bytes(M, K);
}

bl_status bl_forward(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                     int bits, uint16_t* Y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward");
  return forward_common(X, M, K, N, Wp, gamma, bits, Y, bl::kOutBF16, workspace, workspace_bytes, stream);
}

bl_status bl_forward_f32(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                         int bits, float* Y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_f32");
  return forward_common(X, M, K, N, Wp, gamma, bits, Y, bl::kOutF32, workspace, workspace_bytes, stream);
}

size_t bl_matmul_i32_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (check_shape_nk(N, K) != BL_OK || check_m(M, K) != BL_OK) return 0;
  if (M <= kGemvMaxM) return 0;
  return align_up(static_cast<size_t>(M) * 4, 256);
}

bl_status bl_matmul_i32(const int8_t* Xq, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, int32_t* acc,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_matmul_i32");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (M == 0) return BL_OK;
  if (!Xq || !Wp || !acc) return BL_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(Wp)) return BL_ERR_ALIGNMENT;
  const size_t need = bl_matmul_i32_workspace_bytes(M, K, N);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  }
  const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
  if (M <= kGemvMaxM) return launch_gemv(Xq, 1, m, k, n, Wp, nullptr, 0, acc, bl::kOutI32, stream);
  int* R = static_cast<int*>(workspace);
  bl::bl_act_rowsum_kernel<<<(m + bl::kActRowsPerBlock - 1) / bl::kActRowsPerBlock, 256, 0, stream>>>(Xq, m, k, R);
  if ((st = last_cuda()) != BL_OK) return st;
  return launch_tc(Xq, m, k, n, Wp, R, nullptr, nullptr, acc, bl::kOutI32, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free forward: the tensor-core path's scratch lives in one static
// device array (one copy per GPU that loads the library, until exit) instead
// of a caller workspace.  For callers that cannot allocate device memory or
// pass a workspace, e.g. engines that budget all memory at start-up and give an
// operator only its inputs and outputs.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {
constexpr size_t kNoAllocCodeBytes = size_t(16) << 20;    // int8 codes: M*K <= 16 MiB
constexpr int64_t kNoAllocMaxM = 8192;                     // tokens: scales and row sums
constexpr size_t kNoAllocBytes = kNoAllocCodeBytes + 2 * sizeof(int32_t) * kNoAllocMaxM;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::atomic<void*> g_noalloc_addr[kMaxDevices];

// The array's device address on the current device.  Host code must not use
// the symbol itself (it names a host-side stand-in); the address is looked up
// once per device with that device current, then cached.
bl_status noalloc_scratch(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
  void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BL_ERR_CUDA;
    g_noalloc_addr[dev].store(p, std::memory_order_release);
  }
  *out = static_cast<unsigned char*>(p);
  return BL_OK;
}
}  // namespace

extern "C" {

bl_status bl_forward_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp,
                             const float* gamma, int bits, uint16_t* Y, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_noalloc");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!X || !Wp || !gamma || !Y) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wp)) return BL_ERR_ALIGNMENT;
  const int Q = bits == 8 ? 127 : 7;
  const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
  if (M <= kGemvMaxM) return launch_gemv(X, 0, m, k, n, Wp, gamma, Q, Y, bl::kOutBF16, stream);
  if (static_cast<size_t>(M) * static_cast<size_t>(K) > kNoAllocCodeBytes || M > kNoAllocMaxM)
    return BL_ERR_SCRATCH_LIMIT;
  unsigned char* base = nullptr;
  if ((st = noalloc_scratch(&base)) != BL_OK) return st;
  int8_t* Xq = reinterpret_cast<int8_t*>(base);
  float* s = reinterpret_cast<float*>(base + kNoAllocCodeBytes);
  int* R = reinterpret_cast<int*>(base + kNoAllocCodeBytes + sizeof(float) * kNoAllocMaxM);
  // the same activation quantiser choice and GEMM as bl_forward
  if ((st = launch_act_quant(X, m, k, Q, Xq, s, R, stream)) != BL_OK) return st;
  return launch_tc(Xq, m, k, n, Wp, R, s, gamma, Y, bl::kOutBF16, stream);
}

size_t bl_forward_grouped_workspace_bytes(int count, const bl_linear* problems, int bits) {
  (void)bits;
  if (count <= 0 || count > bl::kG2MaxProblems || problems == nullptr) return 0;
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    if (check_shape_nk(p.N, p.K) != BL_OK || check_m(p.M, p.K) != BL_OK) return 0;
    const size_t w = fwd_ws_bytes(p.M, p.K);
    if (w > need) need = w;
  }
  return need;
}

bl_status bl_forward_grouped(int count, const bl_linear* problems, int bits, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_grouped");
  if (problems == nullptr) return BL_ERR_INVALID_ARG;
  if (count < 0 || count > bl::kG2MaxProblems) return BL_ERR_UNSUPPORTED;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  // validate everything before launching anything
  bool all_decode = true;
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    bl_status st = check_shape_nk(p.N, p.K);
    if (st != BL_OK) return st;
    if ((st = check_m(p.M, p.K)) != BL_OK) return st;
    if (p.M == 0) continue;
    if (!p.X || !p.Wp || !p.gamma || !p.Y) return BL_ERR_INVALID_ARG;
    if (!aligned16(p.X) || !aligned16(p.Wp)) return BL_ERR_ALIGNMENT;
    const size_t need = fwd_ws_bytes(p.M, p.K);
    if (need > 0) {
      if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
      if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
    }
    if (p.M != 1 || p.K > 8192) all_decode = false;
  }
  const int Q = bits == 8 ? 127 : 7;
  if (all_decode) {
    // every one-token problem of the call in one launch (any mix of K)
    const bl_linear* sel[bl::kG2MaxProblems];
    int n = 0;
    for (int i = 0; i < count; ++i)
      if (problems[i].M != 0) sel[n++] = &problems[i];
    return launch_decode(sel, n, bl::kInBF16, Q, bl::kOutBF16, stream);
  }
  // otherwise the problems run one after another on the stream (the
  // workspace is reused: stream order serialises them); two problems with
  // more than two tokens that read the same X (same pointer, M and K, e.g.
  // the up and gate projections) share one activation quantisation and, for
  // M > 64, one tensor-core launch over both weight tensors
  bool done_p[bl::kG2MaxProblems] = {};
  for (int i = 0; i < count; ++i) {
    if (done_p[i]) continue;
    const bl_linear& p = problems[i];
    int j = -1;
    if (p.M > kGemvMaxM)
      for (int k = i + 1; k < count && j < 0; ++k)
        if (!done_p[k] && problems[k].X == p.X && problems[k].M == p.M && problems[k].K == p.K) j = k;
    if (j < 0) {
      const bl_status st = forward_common(p.X, p.M, p.K, p.N, p.Wp, p.gamma, bits, p.Y, bl::kOutBF16, workspace,
                                          workspace_bytes, stream);
      if (st != BL_OK) return st;
      continue;
    }
    done_p[j] = true;
    const bl_linear& p2 = problems[j];
    const int m = static_cast<int>(p.M), k = static_cast<int>(p.K);
    const FwdWs w = fwd_ws_split(workspace, p.M, p.K);
    bl_status st = launch_act_quant(p.X, m, k, Q, w.Xq, w.s, w.R, stream);
    if (st != BL_OK) return st;
    if (p.M > 64) {
      const TcProb tp[2] = {{p.Wp, p.gamma, p.Y, static_cast<int>(p.N), nullptr},
                            {p2.Wp, p2.gamma, p2.Y, static_cast<int>(p2.N), nullptr}};
      st = launch_tc_pair_multi(w.Xq, m, k, tp, 2, w.R, w.s, bl::kOutBF16, stream);
    } else {
      st = launch_tc(w.Xq, m, k, static_cast<int>(p.N), p.Wp, w.R, w.s, p.gamma, p.Y, bl::kOutBF16, stream);
      if (st == BL_OK)
        st = launch_tc(w.Xq, m, k, static_cast<int>(p2.N), p2.Wp, w.R, w.s, p2.gamma, p2.Y, bl::kOutBF16, stream);
    }
    if (st != BL_OK) return st;
  }
  return BL_OK;
}

// ---------------------------------------------------------------------------
// Grouped forward on host-resident activations (end to end on one stream).
// ---------------------------------------------------------------------------

// Device staging of a host-buffer group.  Distinct inputs (the same host X
// read by several problems is copied once) and the outputs are sorted by
// host address; host regions that are exactly contiguous form one run,
// staged contiguously (one copy a run), and every run starts 256-byte
// aligned.  Inside a run a tensor keeps its host offset: for inputs a
// multiple of 128 bytes (K % 64 == 0), so staged X stays 16-byte aligned;
// outputs need no alignment.  Only the tensors' own bytes are ever copied.
struct HostRun {
  const uint8_t* host;   // first host byte of the run
  size_t bytes;          // bytes of the run
  size_t stage;          // offset of the run in the staging
};
struct HostStaging {
  size_t x_off[bl::kG2MaxProblems], y_off[bl::kG2MaxProblems];
  HostRun xr[bl::kG2MaxProblems], yr[bl::kG2MaxProblems];
  int nxr = 0, nyr = 0;
  size_t total = 0;
};

// Sort (host pointer, bytes, problem) triples by pointer, cut them into
// exactly contiguous runs from `off` on; returns the offset after the runs.
size_t host_runs(const uint8_t* const* ptr, const size_t* bytes, int m, HostRun* runs, int* nruns, size_t* stage_of,
                 size_t off) {
  int order[bl::kG2MaxProblems];
  for (int i = 0; i < m; ++i) order[i] = i;
  for (int i = 1; i < m; ++i)
    for (int j = i; j > 0 && ptr[order[j]] < ptr[order[j - 1]]; --j) std::swap(order[j], order[j - 1]);
  int r = -1;
  for (int t = 0; t < m; ++t) {
    const int i = order[t];
    if (r < 0 || runs[r].host + runs[r].bytes != ptr[i]) {
      if (r >= 0) off += align_up(runs[r].bytes, 256);
      ++r;
      runs[r] = HostRun{ptr[i], 0, off};
    }
    stage_of[i] = runs[r].stage + static_cast<size_t>(ptr[i] - runs[r].host);
    runs[r].bytes += bytes[i];
  }
  if (r >= 0) off += align_up(runs[r].bytes, 256);
  *nruns = r + 1;
  return off;
}

// Returns false on a bad shape.
bool host_staging_layout(int count, const bl_linear* problems, HostStaging* st) {
  const uint8_t* xp[bl::kG2MaxProblems];
  size_t xb[bl::kG2MaxProblems], xs[bl::kG2MaxProblems];
  int xi[bl::kG2MaxProblems], first[bl::kG2MaxProblems];
  int m = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    if (check_shape_nk(p.N, p.K) != BL_OK || check_m(p.M, p.K) != BL_OK) return false;
    first[i] = -1;
    for (int j = 0; j < i; ++j)
      if (problems[j].X == p.X && problems[j].M == p.M && problems[j].K == p.K) {
        first[i] = first[j] >= 0 ? first[j] : j;
        break;
      }
    if (first[i] < 0) {
      xp[m] = reinterpret_cast<const uint8_t*>(p.X);
      xb[m] = static_cast<size_t>(p.M) * p.K * 2;
      xi[i] = m++;
    }
  }
  size_t off = host_runs(xp, xb, m, st->xr, &st->nxr, xs, 0);
  for (int i = 0; i < count; ++i) st->x_off[i] = xs[xi[first[i] >= 0 ? first[i] : i]];
  const uint8_t* yp[bl::kG2MaxProblems];
  size_t yb[bl::kG2MaxProblems];
  for (int i = 0; i < count; ++i) {
    yp[i] = reinterpret_cast<const uint8_t*>(problems[i].Y);
    yb[i] = static_cast<size_t>(problems[i].M) * problems[i].N * 2;
  }
  off = host_runs(yp, yb, count, st->yr, &st->nyr, st->y_off, off);
  st->total = off;
  return true;
}

// The device address of pinned host memory the device can address, else null.
const uint8_t* host_dev_ptr(const void* host) {
  cudaPointerAttributes a{};
  const uint8_t* d = nullptr;
  if (cudaPointerGetAttributes(&a, host) == cudaSuccess && a.type == cudaMemoryTypeHost && a.devicePointer)
    d = static_cast<const uint8_t*>(a.devicePointer);
  (void)cudaGetLastError();
  return d;
}

// One host-buffer run: a copy kernel when the run is small (the copy
// engine's fixed latency dominates), the host side is pinned memory the
// device can address and both sides are 16-byte aligned; else a copy-engine
// transfer (which also keeps large transfers off the SMs).  h2d: host ->
// staging.
constexpr size_t kCopyKernelMaxBytes = size_t(1) << 20;
bl_status copy_run(const uint8_t* host, uint8_t* stage, size_t bytes, bool h2d, cudaStream_t stream) {
  const uint8_t* hdev = bytes <= kCopyKernelMaxBytes ? host_dev_ptr(host) : nullptr;
  if (hdev == nullptr || !aligned16(hdev) || !aligned16(stage)) {
    if (cudaMemcpyAsync(h2d ? static_cast<void*>(stage) : const_cast<uint8_t*>(host), h2d ? static_cast<const void*>(host) : stage,
                        bytes, h2d ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost, stream) != cudaSuccess) {
      (void)cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return BL_OK;
  }
  const size_t n16 = bytes >> 4;
  const unsigned grid = static_cast<unsigned>(std::max<size_t>(1, std::min<size_t>((n16 + 255) / 256, 148)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* src = h2d ? hdev : stage;
  uint8_t* dst = h2d ? stage : const_cast<uint8_t*>(hdev);
  if (cudaLaunchKernelEx(&cfg, bl::bl_copy_run_kernel, src, dst, bytes) != cudaSuccess) return BL_ERR_CUDA;
  return last_cuda();
}

size_t bl_forward_grouped_host_staging_bytes(int count, const bl_linear* problems) {
  if (count <= 0 || count > bl::kG2MaxProblems || problems == nullptr) return 0;
  HostStaging st;
  return host_staging_layout(count, problems, &st) ? st.total : 0;
}

bl_status bl_forward_grouped_host(int count, const bl_linear* problems, int bits, void* staging, size_t staging_bytes,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_grouped_host");
  if (problems == nullptr) return BL_ERR_INVALID_ARG;
  if (count < 0 || count > bl::kG2MaxProblems) return BL_ERR_UNSUPPORTED;
  if (count == 0) return BL_OK;
  for (int i = 0; i < count; ++i)
    if (problems[i].M == 0 || !problems[i].X || !problems[i].Y) return BL_ERR_INVALID_ARG;
  HostStaging st;
  if (!host_staging_layout(count, problems, &st)) return BL_ERR_SHAPE;
  if (!staging || staging_bytes < st.total) return BL_ERR_WORKSPACE;
  if (!aligned16(staging)) return BL_ERR_ALIGNMENT;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  // outputs may not overlap each other or an input
  for (int i = 0; i < count; ++i) {
    const uint8_t* y0 = reinterpret_cast<const uint8_t*>(problems[i].Y);
    const uint8_t* y1 = y0 + static_cast<size_t>(problems[i].M) * problems[i].N * 2;
    for (int j = 0; j < count; ++j) {
      const uint8_t* x0 = reinterpret_cast<const uint8_t*>(problems[j].X);
      const uint8_t* x1 = x0 + static_cast<size_t>(problems[j].M) * problems[j].K * 2;
      if (y0 < x1 && x0 < y1) return BL_ERR_INVALID_ARG;
      if (j != i) {
        const uint8_t* z0 = reinterpret_cast<const uint8_t*>(problems[j].Y);
        const uint8_t* z1 = z0 + static_cast<size_t>(problems[j].M) * problems[j].N * 2;
        if (y0 < z1 && z0 < y1) return BL_ERR_INVALID_ARG;
      }
    }
  }
  bl_linear dev[bl::kG2MaxProblems];
  uint8_t* base = static_cast<uint8_t*>(staging);
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    if (!p.Wp || !p.gamma) return BL_ERR_INVALID_ARG;
    if (!aligned16(p.Wp)) return BL_ERR_ALIGNMENT;
    const size_t w = fwd_ws_bytes(p.M, p.K);
    if (w > 0 && (!workspace || workspace_bytes < w)) return BL_ERR_WORKSPACE;
    if (w > 0 && !aligned16(workspace)) return BL_ERR_ALIGNMENT;
    dev[i] = p;
    dev[i].X = reinterpret_cast<const uint16_t*>(base + st.x_off[i]);
    dev[i].Y = reinterpret_cast<uint16_t*>(base + st.y_off[i]);
  }
  bl_status rc;
  for (int r = 0; r < st.nxr; ++r)
    if ((rc = copy_run(st.xr[r].host, base + st.xr[r].stage, st.xr[r].bytes, true, stream)) != BL_OK) return rc;
  rc = bl_forward_grouped(count, dev, bits, workspace, workspace_bytes, stream);
  if (rc != BL_OK) return rc;
  for (int r = 0; r < st.nyr; ++r)
    if ((rc = copy_run(st.yr[r].host, base + st.yr[r].stage, st.yr[r].bytes, false, stream)) != BL_OK) return rc;
  return BL_OK;
}

size_t relu2_ws_bytes(int64_t M, int64_t K) {
  if (M == 1 && K <= 8192) return 0;   // the decode kernels quantise in their prologue
  return align_up(static_cast<size_t>(M) * K, 256) + 2 * align_up(static_cast<size_t>(M) * 4, 256);
}

size_t bl_forward_relu2_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  (void)bits;
  if (check_shape_nk(N, K) != BL_OK || check_m(M, K) != BL_OK || M == 0) return 0;
  return relu2_ws_bytes(M, K);
}

bl_status bl_quant_act_relu2(const uint16_t* G, const uint16_t* U, int64_t M, int64_t K, int bits, int8_t* Xq,
                             float* scale, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quant_act_relu2");
  if (K <= 0 || (K % 64) != 0 || K > kMaxK) return BL_ERR_SHAPE;
  bl_status st = check_m(M, K);
  if (st != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!G || !Xq || !scale) return BL_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(Xq) || (U && !aligned16(U))) return BL_ERR_ALIGNMENT;
  bl::bl_act_quant_relu2_kernel<<<static_cast<unsigned>(M), bl::kActRowThreads, 0, stream>>>(
      G, U, U != nullptr, static_cast<int>(K), bits == 8 ? 127 : 7, Xq, scale, nullptr);
  return last_cuda();
}

bl_status bl_forward_relu2(const uint16_t* G, const uint16_t* U, int64_t M, int64_t K, int64_t N, const uint8_t* Wp,
                           const float* gamma, int bits, uint16_t* Y, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_relu2");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!G || !Wp || !gamma || !Y) return BL_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(Wp) || (U && !aligned16(U))) return BL_ERR_ALIGNMENT;
  const size_t need = relu2_ws_bytes(M, K);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  }
  const int Q = bits == 8 ? 127 : 7;
  if (need == 0) {   // one token: squared ReLU and quantisation in the decode kernel's prologue
    bl_linear p;
    p.X = G;
    p.M = 1;
    p.K = K;
    p.N = N;
    p.Wp = Wp;
    p.gamma = gamma;
    p.Y = Y;
    const bl_linear* pp = &p;
    const void* us[1] = {U};
    return launch_decode(&pp, 1, U ? bl::kInRelu2Gated : bl::kInRelu2, Q, bl::kOutBF16, stream, us);
  }
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int8_t* Xq = reinterpret_cast<int8_t*>(base);
  float* s = reinterpret_cast<float*>(base + align_up(static_cast<size_t>(M) * K, 256));
  int* R = reinterpret_cast<int*>(base + align_up(static_cast<size_t>(M) * K, 256) +
                                  align_up(static_cast<size_t>(M) * 4, 256));
  bl::bl_act_quant_relu2_kernel<<<static_cast<unsigned>(M), bl::kActRowThreads, 0, stream>>>(
      G, U, U != nullptr, static_cast<int>(K), Q, Xq, s, R);
  if ((st = last_cuda()) != BL_OK) return st;
  return launch_tc(Xq, static_cast<int>(M), static_cast<int>(K), static_cast<int>(N), Wp, R, s, gamma, Y, bl::kOutBF16,
                   stream);
}

size_t ex_ws_bytes(int64_t M, int64_t K) {
  if (M == 1 && K <= 8192) return 0;   // one token: the decode kernels, no workspace
  return align_up(static_cast<size_t>(M) * K, 256) + 2 * align_up(static_cast<size_t>(M) * 4, 256) + 256;
}

size_t bl_forward_ex_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits, unsigned flags) {
  (void)bits;
  (void)flags;
  if (check_shape_nk(N, K) != BL_OK || check_m(M, K) != BL_OK || M == 0) return 0;
  return ex_ws_bytes(M, K);
}

bl_status bl_forward_ex(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                        int bits, unsigned flags, const float* bias, uint16_t* Y, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_ex");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if ((flags & ~static_cast<unsigned>(BL_ACT_PER_TENSOR)) != 0u) return BL_ERR_UNSUPPORTED;
  if (M == 0) return BL_OK;
  if (!X || !Wp || !gamma || !Y) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wp) || (reinterpret_cast<uintptr_t>(bias) & 3u)) return BL_ERR_ALIGNMENT;
  const size_t need = ex_ws_bytes(M, K);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  }
  const int Q = bits == 8 ? 127 : 7;
  if (need == 0) {   // one token: per-tensor and per-token scales coincide
    bl_linear p;
    p.X = X;
    p.M = 1;
    p.K = K;
    p.N = N;
    p.Wp = Wp;
    p.gamma = gamma;
    p.Y = Y;
    const bl_linear* pp = &p;
    return launch_decode(&pp, 1, bl::kInBF16, Q, bl::kOutBF16, stream, nullptr, bias);
  }
  const int m = static_cast<int>(M), k = static_cast<int>(K);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const size_t codes = align_up(static_cast<size_t>(M) * K, 256), rows = align_up(static_cast<size_t>(M) * 4, 256);
  int8_t* Xq = reinterpret_cast<int8_t*>(base);
  float* s = reinterpret_cast<float*>(base + codes);
  int* R = reinterpret_cast<int*>(base + codes + rows);
  uint32_t* amax = reinterpret_cast<uint32_t*>(base + codes + 2 * rows);
  if (flags & BL_ACT_PER_TENSOR) {
    if (cudaMemsetAsync(amax, 0, sizeof(uint32_t), stream) != cudaSuccess) return BL_ERR_CUDA;
    const int64_t nch = static_cast<int64_t>(M) * K / 8;
    int64_t blocks = (nch + 255) / 256;
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    bl::bl_act_absmax_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(X, nch, amax);
    if ((st = last_cuda()) != BL_OK) return st;
    bl::bl_act_quant_row_kernel<false><<<m, bl::kActRowThreads, 0, stream>>>(X, k, Q, Xq, s, R, amax);
    if ((st = last_cuda()) != BL_OK) return st;
  } else if ((st = launch_act_quant(X, m, k, Q, Xq, s, R, stream)) != BL_OK) {
    return st;
  }
  return launch_tc(Xq, m, k, static_cast<int>(N), Wp, R, s, gamma, Y, bl::kOutBF16, stream, bias);
}

size_t rms_ws_bytes(int64_t M, int64_t K) {
  return align_up(static_cast<size_t>(M) * K, 256) + 3 * align_up(static_cast<size_t>(M) * 4, 256);
}

size_t bl_forward_rmsnorm_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  (void)bits;
  if (check_shape_nk(N, K) != BL_OK || check_m(M, K) != BL_OK || M == 0) return 0;
  return rms_ws_bytes(M, K);
}

size_t bl_forward_layernorm_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  return bl_forward_rmsnorm_workspace_bytes(M, K, N, bits);
}

bool rms_eps_ok(float eps) { return eps > 0.f && std::isfinite(eps); }

// The normalising quantiser (one CTA per token): RMSNorm with an optional
// weight, or LayerNorm.  st0: ms (RMSNorm) or mean (LayerNorm); st1: var.
bl_status launch_norm_quant(int norm, const uint16_t* X, const uint16_t* w, float eps, int m, int k, int Q,
                            int8_t* Xq, float* s, int* R, float* st0, float* st1, cudaStream_t stream) {
  if (norm == BL_NORM_LAYER)
    bl::bl_act_quant_norm_kernel<bl::kNormLayer><<<static_cast<unsigned>(m), bl::kActRowThreads, 0, stream>>>(
        X, nullptr, eps, k, Q, Xq, s, R, st0, st1);
  else
    bl::bl_act_quant_norm_kernel<bl::kNormRms><<<static_cast<unsigned>(m), bl::kActRowThreads, 0, stream>>>(
        X, w, eps, k, Q, Xq, s, R, st0, nullptr);
  return last_cuda();
}

// Whether one-token problems go through one resident decode launch with the
// normalising prologue (K <= 8192 each, all weights within the SMs' rings).
bool norm_decode_fits(const bl_linear* const* probs, int n) {
  double wbytes = 0.0;
  for (int i = 0; i < n; ++i) {
    if (probs[i]->M != 1 || probs[i]->K > bl::kDecMaxK) return false;
    wbytes += static_cast<double>(probs[i]->N) * static_cast<double>(probs[i]->K) / 4.0;
  }
  return wbytes <= static_cast<double>(num_sms()) * bl::kDecRingBytes;
}

// One normalised BitLinear forward (arguments validated by the caller).
bl_status forward_norm(int norm, const uint16_t* X, const uint16_t* w, float eps, int64_t M, int64_t K, int64_t N,
                       const uint8_t* Wp, const float* gamma, int bits, uint16_t* Y, void* workspace,
                       cudaStream_t stream) {
  const int Q = bits == 8 ? 127 : 7;
  bl_linear p;
  p.X = X;
  p.M = M;
  p.K = K;
  p.N = N;
  p.Wp = Wp;
  p.gamma = gamma;
  p.Y = Y;
  const bl_linear* pp = &p;
  if (norm_decode_fits(&pp, 1)) {
    // one token whose layer fits the resident decode kernel: normalisation,
    // absmax and quantisation in its prologue (the workspace stays unused)
    const void* us[1] = {w};
    return launch_decode(&pp, 1, norm == BL_NORM_LAYER ? bl::kInLayerNorm : bl::kInRmsNorm, Q, bl::kOutBF16, stream,
                         us, nullptr, eps);
  }
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const size_t codes = align_up(static_cast<size_t>(M) * K, 256), rows = align_up(static_cast<size_t>(M) * 4, 256);
  int8_t* Xq = reinterpret_cast<int8_t*>(base);
  float* s = reinterpret_cast<float*>(base + codes);
  int* R = reinterpret_cast<int*>(base + codes + rows);
  bl_status st = launch_norm_quant(norm, X, w, eps, static_cast<int>(M), static_cast<int>(K), Q, Xq, s, R, nullptr,
                                   nullptr, stream);
  if (st != BL_OK) return st;
  return launch_tc(Xq, static_cast<int>(M), static_cast<int>(K), static_cast<int>(N), Wp, R, s, gamma, Y,
                   bl::kOutBF16, stream);
}

// Shared validation of the normalising quantiser exports.
bl_status check_norm_quant(const uint16_t* X, const uint16_t* w, float eps, int64_t M, int64_t K, int bits,
                           const int8_t* Xq, const float* scale, const float* st0, const float* st1) {
  if (K <= 0 || (K % 64) != 0 || K > kMaxK) return BL_ERR_SHAPE;
  bl_status st = check_m(M, K);
  if (st != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (!rms_eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!X || !Xq || !scale) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq) || (w && !aligned16(w)) || (reinterpret_cast<uintptr_t>(st0) & 3u) ||
      (reinterpret_cast<uintptr_t>(st1) & 3u))
    return BL_ERR_ALIGNMENT;
  return BL_OK;
}

bl_status bl_quant_act_rmsnorm(const uint16_t* X, const uint16_t* norm_weight, float eps, int64_t M, int64_t K,
                               int bits, int8_t* Xq, float* scale, float* mean_sq, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quant_act_rmsnorm");
  const bl_status st = check_norm_quant(X, norm_weight, eps, M, K, bits, Xq, scale, mean_sq, nullptr);
  if (st != BL_OK || M == 0) return st;
  return launch_norm_quant(BL_NORM_RMS, X, norm_weight, eps, static_cast<int>(M), static_cast<int>(K),
                           bits == 8 ? 127 : 7, Xq, scale, nullptr, mean_sq, nullptr, stream);
}

bl_status bl_quant_act_layernorm(const uint16_t* X, float eps, int64_t M, int64_t K, int bits, int8_t* Xq,
                                 float* scale, float* mean, float* var, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quant_act_layernorm");
  const bl_status st = check_norm_quant(X, nullptr, eps, M, K, bits, Xq, scale, mean, var);
  if (st != BL_OK || M == 0) return st;
  return launch_norm_quant(BL_NORM_LAYER, X, nullptr, eps, static_cast<int>(M), static_cast<int>(K),
                           bits == 8 ? 127 : 7, Xq, scale, nullptr, mean, var, stream);
}

// Shared validation of one normalised forward problem.
bl_status check_norm_forward(const uint16_t* X, const uint16_t* w, float eps, int64_t M, int64_t K, int64_t N,
                             const uint8_t* Wp, const float* gamma, int bits, const uint16_t* Y, const void* workspace,
                             size_t workspace_bytes) {
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  if (!rms_eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!X || !Wp || !gamma || !Y) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wp) || (w && !aligned16(w))) return BL_ERR_ALIGNMENT;
  const size_t need = rms_ws_bytes(M, K);
  if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  return BL_OK;
}

bl_status bl_forward_rmsnorm(const uint16_t* X, const uint16_t* norm_weight, float eps, int64_t M, int64_t K,
                             int64_t N, const uint8_t* Wp, const float* gamma, int bits, uint16_t* Y,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_rmsnorm");
  const bl_status st =
      check_norm_forward(X, norm_weight, eps, M, K, N, Wp, gamma, bits, Y, workspace, workspace_bytes);
  if (st != BL_OK || M == 0) return st;
  return forward_norm(BL_NORM_RMS, X, norm_weight, eps, M, K, N, Wp, gamma, bits, Y, workspace, stream);
}

bl_status bl_forward_layernorm(const uint16_t* X, float eps, int64_t M, int64_t K, int64_t N, const uint8_t* Wp,
                               const float* gamma, int bits, uint16_t* Y, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_layernorm");
  const bl_status st = check_norm_forward(X, nullptr, eps, M, K, N, Wp, gamma, bits, Y, workspace, workspace_bytes);
  if (st != BL_OK || M == 0) return st;
  return forward_norm(BL_NORM_LAYER, X, nullptr, eps, M, K, N, Wp, gamma, bits, Y, workspace, stream);
}

size_t bl_forward_norm_grouped_workspace_bytes(int count, const bl_linear* problems, int bits) {
  (void)bits;
  if (!problems || count < 0 || count > bl::kG2MaxProblems) return 0;
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    if (check_shape_nk(p.N, p.K) != BL_OK || check_m(p.M, p.K) != BL_OK) return 0;
    if (p.M != 0) need = std::max(need, rms_ws_bytes(p.M, p.K));
  }
  return need;
}

bl_status bl_forward_norm_grouped(int count, const bl_linear* problems, int norm, const uint16_t* const* norm_weights,
                                  float eps, int bits, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_norm_grouped");
  if (problems == nullptr) return BL_ERR_INVALID_ARG;
  if (count < 0 || count > bl::kG2MaxProblems) return BL_ERR_UNSUPPORTED;
  if (norm != BL_NORM_RMS && norm != BL_NORM_LAYER) return BL_ERR_UNSUPPORTED;
  if (norm == BL_NORM_LAYER && norm_weights != nullptr) return BL_ERR_INVALID_ARG;
  // validate everything before launching anything
  const bl_linear* sel[bl::kG2MaxProblems];
  const void* us[bl::kG2MaxProblems];
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear& p = problems[i];
    const uint16_t* w = norm_weights ? norm_weights[i] : nullptr;
    const bl_status st = check_norm_forward(static_cast<const uint16_t*>(p.X), w, eps, p.M, p.K, p.N, p.Wp, p.gamma,
                                            bits, static_cast<const uint16_t*>(p.Y), workspace, workspace_bytes);
    if (st != BL_OK) return st;
    if (p.M == 0) continue;
    sel[n] = &p;
    us[n++] = w;
  }
  if (n == 0) return BL_OK;
  if (norm_decode_fits(sel, n)) {
    // every one-token problem of the call in one launch, each CTA normalising
    // its own problem's token
    return launch_decode(sel, n, norm == BL_NORM_LAYER ? bl::kInLayerNorm : bl::kInRmsNorm, bits == 8 ? 127 : 7,
                         bl::kOutBF16, stream, us, nullptr, eps);
  }
  for (int i = 0; i < n; ++i) {
    const bl_linear& p = *sel[i];
    const bl_status st = forward_norm(norm, static_cast<const uint16_t*>(p.X), static_cast<const uint16_t*>(us[i]),
                                      eps, p.M, p.K, p.N, p.Wp, p.gamma, bits, static_cast<uint16_t*>(p.Y), workspace,
                                      stream);
    if (st != BL_OK) return st;
  }
  return BL_OK;
}

// ---------------------------------------------------------------------------
// Base-3 weight storage (five weights a byte; see bl_weights.cuh).
// ---------------------------------------------------------------------------

size_t bl_packed_weight_bytes_b3(int64_t N, int64_t K) {
  if (check_shape_nk(N, K) != BL_OK) return 0;
  return static_cast<size_t>(N) * 4u * static_cast<size_t>(bl::base3_row_words(static_cast<int>(K)));
}

bl_status bl_quantize_weights_b3(const float* W, int64_t N, int64_t K, uint8_t* Wp3, float* gamma, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_quantize_weights_b3");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if (N > INT32_MAX) return BL_ERR_SHAPE;
  if (!W || !Wp3 || !gamma) return BL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wp3)) return BL_ERR_ALIGNMENT;
  const size_t need = bl_quantize_weights_workspace_bytes(N, K);
  if (!workspace || workspace_bytes < need) return BL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BL_ERR_ALIGNMENT;
  auto* bins = static_cast<unsigned long long*>(workspace);
  const int64_t n = N * K;
  if (cudaMemsetAsync(bins, 0, bl::kAbsumTotals * sizeof(unsigned long long), stream) != cudaSuccess)
    return BL_ERR_CUDA;
  bl::bl_weight_absum_kernel<<<absum_blocks(N, K), bl::kAbsumThreads, 0, stream>>>(W, n, bins);
  if ((st = last_cuda()) != BL_OK) return st;
  bl::bl_weight_gamma_kernel<<<1, 32, 0, stream>>>(bins, static_cast<uint64_t>(n), gamma);
  if ((st = last_cuda()) != BL_OK) return st;
  const int64_t nwords = N * bl::base3_row_words(static_cast<int>(K));
  bl::bl_weight_pack3_kernel<<<static_cast<unsigned>((nwords + 255) / 256), 256, 0, stream>>>(
      W, static_cast<int>(N), static_cast<int>(K), gamma, reinterpret_cast<uint32_t*>(Wp3));
  return last_cuda();
}

bl_status bl_unpack_weights_b3(const uint8_t* Wp3, int64_t N, int64_t K, int8_t* codes, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_unpack_weights_b3");
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if (N > INT32_MAX) return BL_ERR_SHAPE;
  if (!Wp3 || !codes) return BL_ERR_INVALID_ARG;
  if (!aligned16(Wp3)) return BL_ERR_ALIGNMENT;
  const int64_t nwords = N * bl::base3_row_words(static_cast<int>(K));
  bl::bl_weight_unpack3_kernel<<<static_cast<unsigned>((nwords + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(Wp3), static_cast<int>(N), static_cast<int>(K), codes);
  return last_cuda();
}

}  // extern "C"

namespace {
// One token on base-3 weights: the resident decode kernel in its base-3 form.
bl_status forward_b3_common(const void* X, int in_mode, int64_t M, int64_t K, int64_t N, const uint8_t* Wp3,
                            const float* gamma, int Q, void* Y, int out_mode, cudaStream_t stream) {
  bl_status st = check_shape_nk(N, K);
  if (st != BL_OK) return st;
  if ((st = check_m(M, K)) != BL_OK) return st;
  if (M == 0) return BL_OK;
  if (M != 1 || K > bl::kDecMaxK || N > INT32_MAX) return BL_ERR_UNSUPPORTED;
  if (!X || !Wp3 || !Y || (out_mode != bl::kOutI32 && !gamma)) return BL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wp3)) return BL_ERR_ALIGNMENT;
  bl_linear p;
  p.X = static_cast<const uint16_t*>(X);
  p.M = 1;
  p.K = K;
  p.N = N;
  p.Wp = Wp3;
  p.gamma = gamma;
  p.Y = static_cast<uint16_t*>(Y);
  const bl_linear* pp = &p;
  const int sms = num_sms();
  const bool big = static_cast<double>(N) * dec_row_bytes(K, bl::kFmtBase3) > static_cast<double>(sms) * bl::kDecRingBytes;
  bl::G2Table tab;
  const int mode = big ? bl::kModeBig : bl::kModeResident;
  const int grid = fill_decode_table(&tab, &pp, 1, sms, mode, 0, nullptr, nullptr, 0.f, bl::kFmtBase3);
  if (big)
    return launch_dec_t<0, bl::kDecPlain, bl::kFmtBase3, bl::kModeBig>(tab, grid, in_mode, Q, out_mode, stream);
  return launch_dec_t<0, bl::kDecPlain, bl::kFmtBase3, bl::kModeResident>(tab, grid, in_mode, Q, out_mode, stream);
}
}  // namespace

extern "C" {

bl_status bl_forward_b3(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp3, const float* gamma,
                        int bits, uint16_t* Y, cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_forward_b3");
  if (bits != 8 && bits != 4) return BL_ERR_UNSUPPORTED;
  return forward_b3_common(X, bl::kInBF16, M, K, N, Wp3, gamma, bits == 8 ? 127 : 7, Y, bl::kOutBF16, stream);
}

bl_status bl_matmul_i32_b3(const int8_t* Xq, int64_t M, int64_t K, int64_t N, const uint8_t* Wp3, int32_t* acc,
                           cudaStream_t stream) {
  const NvtxRange nvtx_range("bl_matmul_i32_b3");
  return forward_b3_common(Xq, bl::kInI8, M, K, N, Wp3, nullptr, 0, acc, bl::kOutI32, stream);
}

// Throughput probe of tcgen05.mma kind::i8 (see bl_probe.cuh).
bl_status bl_probe_mma_i8(int n_mma, int n_cols, unsigned long long* out, int grid, cudaStream_t stream) {
  if (!out) return BL_ERR_INVALID_ARG;
  if (n_mma <= 0 || n_mma > (1 << 22) || grid <= 0 || grid > 4096) return BL_ERR_SHAPE;
  if (n_cols < 16 || n_cols > 256 || (n_cols % 16) != 0) return BL_ERR_SHAPE;
  static std::atomic<uint64_t> done{0};
  if (!ensure_smem(bl::bl_probe_mma_i8_kernel, bl::kProbeSmemBytes, &done)) return BL_ERR_CUDA;
  bl::bl_probe_mma_i8_kernel<<<grid, bl::kProbeThreads, bl::kProbeSmemBytes, stream>>>(n_mma, n_cols, out,
                                                                                       kWaitLimitNs);
  return last_cuda();
}

bl_status bl_probe_mma_i8_pair(int n_mma, int n_cols, unsigned long long* out, int grid, cudaStream_t stream) {
  if (!out) return BL_ERR_INVALID_ARG;
  if (n_mma <= 0 || n_mma > (1 << 22) || grid <= 0 || grid > 4096 || (grid % 2) != 0) return BL_ERR_SHAPE;
  if (n_cols < 32 || n_cols > 256 || (n_cols % 32) != 0) return BL_ERR_SHAPE;
  static std::atomic<uint64_t> done{0};
  if (!ensure_smem(bl::bl_probe_mma_i8_pair_kernel, bl::kProbeSmemBytes, &done)) return BL_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(bl::kProbeThreads);
  cfg.dynamicSmemBytes = bl::kProbeSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const unsigned long long lim = kWaitLimitNs;
  if (cudaLaunchKernelEx(&cfg, bl::bl_probe_mma_i8_pair_kernel, n_mma, n_cols, out, lim) != cudaSuccess)
    return BL_ERR_CUDA;
  return last_cuda();
}

bl_status bl_device_status(int clear, int* site) {
  if (cudaDeviceSynchronize() != cudaSuccess) return BL_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bl::g_status, sizeof(v)) != cudaSuccess) return BL_ERR_CUDA;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(bl::g_status, &z, sizeof(z)) != cudaSuccess) return BL_ERR_CUDA;
  }
  if (site) *site = static_cast<int>((v >> 8) & 0xffu);
  return static_cast<bl_status>(v & 0xffu);
}

bl_status bl_selftest_wait_timeout(unsigned long long limit_ns, int* waited_ok, cudaStream_t stream) {
  if (!waited_ok) return BL_ERR_INVALID_ARG;
  if (limit_ns > 10ull * kWaitLimitNs) return BL_ERR_INVALID_ARG;
  bl::bl_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, waited_ok);
  return last_cuda();
}

// ---------------------------------------------------------------------------
// A host-buffer grouped forward recorded once as a CUDA graph and replayed.
// ---------------------------------------------------------------------------

struct bl_graph_s {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

bl_status bl_forward_grouped_host_graph(int count, const bl_linear* problems, int bits, void* staging,
                                        size_t staging_bytes, void* workspace, size_t workspace_bytes,
                                        cudaStream_t stream, bl_graph* out) {
  const NvtxRange nvtx_range("bl_forward_grouped_host_graph");
  if (out == nullptr) return BL_ERR_INVALID_ARG;
  *out = nullptr;
  if (problems == nullptr) return BL_ERR_INVALID_ARG;
  if (count <= 0 || count > bl::kG2MaxProblems) return BL_ERR_UNSUPPORTED;
  // one plain call first, on the caller's stream (after the caller's work
  // there): it validates the arguments and does the kernels' one-time set-up
  // on this device outside the capture
  bl_status rc = bl_forward_grouped_host(count, problems, bits, staging, staging_bytes, workspace, workspace_bytes,
                                         stream);
  if (rc != BL_OK) return rc;
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return BL_ERR_CUDA;
  }
  cudaStream_t s = nullptr;   // the capture runs on a private stream
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
    (void)cudaGetLastError();
    return BL_ERR_CUDA;
  }
  cudaGraph_t g = nullptr;
  if (rc == BL_OK) {
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      rc = BL_ERR_CUDA;
    } else {
      rc = bl_forward_grouped_host(count, problems, bits, staging, staging_bytes, workspace, workspace_bytes, s);
      if (cudaStreamEndCapture(s, &g) != cudaSuccess && rc == BL_OK) rc = BL_ERR_CUDA;
    }
  }
  cudaGraphExec_t ex = nullptr;
  if (rc == BL_OK && cudaGraphInstantiate(&ex, g, 0) != cudaSuccess) rc = BL_ERR_CUDA;
  bl_graph h = nullptr;
  if (rc == BL_OK) {
    h = new (std::nothrow) bl_graph_s;
    if (h == nullptr) rc = BL_ERR_CUDA;
  }
  if (rc != BL_OK) {
    (void)cudaGetLastError();
    if (ex) cudaGraphExecDestroy(ex);
    if (g) cudaGraphDestroy(g);
    cudaStreamDestroy(s);
    return rc;
  }
  h->graph = g;
  h->exec = ex;
  cudaStreamDestroy(s);
  *out = h;
  return BL_OK;
}

bl_status bl_graph_launch(bl_graph graph, cudaStream_t stream) {
  if (graph == nullptr) return BL_ERR_INVALID_ARG;
  if (cudaGraphLaunch(graph->exec, stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return BL_ERR_CUDA;
  }
  return BL_OK;
}

void bl_graph_destroy(bl_graph graph) {
  if (graph == nullptr) return;
  if (graph->exec) cudaGraphExecDestroy(graph->exec);
  if (graph->graph) cudaGraphDestroy(graph->graph);
  delete graph;
}

}  // extern "C"
