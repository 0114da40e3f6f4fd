/*
 * libbitlinear -- BitNet b1.58 BitLinear forward on NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every pointer argument that names a tensor is a DEVICE pointer that
 * the caller allocated and owns.  The library allocates no device memory at
 * run time; its only device memory of its own is static: one 4-byte status
 * word (see bl_device_status) and the 16 MiB + 64 KiB scratch array of
 * bl_forward_noalloc, both present on every GPU that loads the library until
 * the process exits.  Every compute
 * call is asynchronous on the given CUDA stream (0 = legacy default stream)
 * and returns a bl_status:
 *   - arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and leaves every output untouched;
 *   - BL_ERR_CUDA reports a launch failure (cudaGetLastError);
 *   - problems found while a kernel runs (a pipeline wait that gave up) are
 *     recorded in the device status word, read with bl_device_status.
 * Calls on distinct streams are thread-safe.  Inputs containing NaN or Inf
 * give undefined (but memory-safe) results.
 *
 * Notation: X bf16 [M, K] activations (tokens x in-features, row-major),
 * W fp32 [N, K] latent weights (out-features x in-features, the nn.Linear
 * convention), Y [M, N] outputs (row-major).  bf16 tensors are passed as
 * pointers to their 16-bit patterns.
 *
 * Sources (web pages, cited by title and section):
 *   [b1.58] "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide",
 *           section "The Mathematical Formulation of BitLinear", eqs. (1)-(3).
 *   [a4.8]  "BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs", section
 *           "1. Hybrid W1.58 / A4 Quantization Function".
 *   [2B4T]  "BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs", section
 *           "1. The BitLinear Operator".
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = 1, /* null pointer where a tensor is required */
  BL_ERR_SHAPE = 2,       /* M < 0, N or K <= 0, K % 64 != 0, K > 65536, N*K >= 2^40 */
  BL_ERR_ALIGNMENT = 3,   /* a pointer that must be 16-byte aligned is not */
  BL_ERR_UNSUPPORTED = 4, /* bits not in {4, 8} */
  BL_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed */
  BL_ERR_TIMEOUT = 6,     /* a kernel's bounded wait gave up (device status word) */
  BL_ERR_WORKSPACE = 7,   /* workspace pointer null or smaller than required */
  BL_ERR_SCRATCH_LIMIT = 8 /* shape exceeds the built-in scratch of bl_forward_noalloc */
} bl_status;

/* Static, NUL-terminated description of a status code. */
BL_API const char* bl_status_string(bl_status s);

/* Library version as major*10000 + minor*100 + patch. */
BL_API int bl_version(void);

/* ---------------------------------------------------------------------------
 * Packed ternary weights.
 *
 * Storage: 2 bits per weight, N*K/4 bytes (the a4.8 page's verification
 * harness counts in*out*2/8 bytes; the bit layout is this library's).  Row n
 * starts at byte n*K/4 and is a run of little-endian 32-bit words; word g holds
 * weights k = 16g..16g+15; weight k = 16g + 4j + b (j, b in 0..3) sits in bits
 * [8b+2j, 8b+2j+2) and stores code+1 (0 = -1, 1 = 0, 2 = +1; 3 is never
 * written).  gamma is one fp32 in device memory.
 * ------------------------------------------------------------------------- */

/* N*K/4. */
BL_API size_t bl_packed_weight_bytes(int64_t N, int64_t K);

/* Device workspace bytes bl_quantize_weights needs (independent of the data). */
BL_API size_t bl_quantize_weights_workspace_bytes(int64_t N, int64_t K);

/*
 * [b1.58] eq. (1), absmean weight quantisation:
 *   gamma = max(mean_{n,k} |W[n,k]|, 1e-5)   -- the mean is formed exactly
 *           and rounded once to fp32 (nearest, ties to even), so gamma does not
 *           depend on any summation order;
 *   code  = clamp(round_half_even(W / gamma), -1, 1)   (IEEE fp32 division);
 *   Wp    = packed codes (layout above), gamma written to *gamma.
 * W: fp32 [N, K], 16-byte aligned.  Wp: N*K/4 bytes, 16-byte aligned.
 * workspace: at least bl_quantize_weights_workspace_bytes(N, K) bytes,
 * 16-byte aligned, contents ignored and clobbered.
 */
BL_API bl_status bl_quantize_weights(const float* W, int64_t N, int64_t K, uint8_t* Wp, float* gamma, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/* Packed weights -> int8 codes in {-1, 0, 1}, row-major [N, K] (16-byte
 * aligned).  For tests and inspection. */
BL_API bl_status bl_unpack_weights(const uint8_t* Wp, int64_t N, int64_t K, int8_t* codes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Activations.
 * ------------------------------------------------------------------------- */

/*
 * [b1.58] eq. (2) per token, with the [2B4T] clip range and the [a4.8] 4-bit
 * mode.  For each row m of X:
 *   a_m  = max_k |X[m,k]|
 *   s_m  = Q / max(a_m, 1e-5)                     (fp32 division)
 *   q    = clamp(round_half_even(X * s_m), -Q-1, Q)  (fp32 product)
 * with Q = 127 for bits = 8 and Q = 7 for bits = 4.
 * X: bf16 bits [M, K], 16-byte aligned.  Xq: int8 [M, K] (4-bit codes are
 * stored one per byte), 16-byte aligned.  scale: fp32 [M], receives s_m.
 * M == 0 is a no-op.
 */
BL_API bl_status bl_quant_act(const uint16_t* X, int64_t M, int64_t K, int bits, int8_t* Xq, float* scale,
                       cudaStream_t stream);

/*
 * The 4-bit mode of bl_quant_act with the codes packed two a byte ("BitNet
 * a4.8 Guide: 4-Bit Activation 1-Bit LLMs", section "Step 4: Verification and
 * Benchmarking Test Harness": 4-bit activations take n / 2 bytes): the same
 * per-token codes as bl_quant_act(bits = 4) (Q = 7, range [-8, 7]), stored as
 * two's-complement nibbles, code 2j of a row in the low nibble of byte j and
 * code 2j + 1 in its high nibble.  Xq4: [M, K/2] bytes, 16-byte aligned.
 * scale: fp32 [M], receives s_m.  M == 0 is a no-op.
 */
BL_API bl_status bl_quant_act_packed4(const uint16_t* X, int64_t M, int64_t K, uint8_t* Xq4, float* scale,
                                      cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Forward.
 * ------------------------------------------------------------------------- */

/* Device workspace bytes bl_forward / bl_forward_f32 need for this shape (0
 * when the decode path is taken, M <= 2). */
BL_API size_t bl_forward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);

/*
 * [b1.58] eqs. (2)-(3): the BitLinear forward on packed weights.
 *   q, s_m  = per-token activation quantisation of X (see bl_quant_act)
 *   acc     = sum_k q[m,k] * code[n,k]        (exact int32)
 *   Y[m,n]  = bf16_round_nearest_even( f32(acc) * f32(gamma / s_m) )
 * Decode (M <= 2): one fused kernel (quantisation prologue + GEMV).
 * Otherwise: an activation-quantisation kernel writes int8 codes, scales and
 * row sums into the workspace, then a tcgen05 tensor-core GEMM runs.
 * X: bf16 bits [M, K], 16-byte aligned.  Wp, gamma: from bl_quantize_weights.
 * Y: bf16 bits [M, N].  workspace: >= bl_forward_workspace_bytes(M, K, N, bits)
 * bytes, 16-byte aligned (may be null when that is 0).
 * Ordering: the kernels are launched with programmatic dependent launch.  They
 * read X (and the workspace) only after the preceding kernel on the stream has
 * completed, but a one-token launch may fetch Wp and gamma before that, while
 * the preceding kernel still runs: neither may be written by the kernel launched
 * immediately before on the same stream if that kernel triggers its dependents
 * early (this library's forward kernels do; bl_quantize_weights and ordinary
 * kernels do not, and a dependent launch after them starts only once they
 * have finished).
 */
BL_API bl_status bl_forward(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                     int bits, uint16_t* Y, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* As bl_forward but writes the fp32 value f32(acc) * f32(gamma / s_m) before
 * the bf16 rounding.  For tests. */
BL_API bl_status bl_forward_f32(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, const float* gamma,
                         int bits, float* Y, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Allocation-free forward.  The pages have no counterpart of this call; it is
 * an integration aid.  Some callers cannot allocate device memory or hand the
 * library a workspace: for example an engine that budgets all device memory
 * once at start-up and gives its operators only their input and output
 * buffers, or a plug-in whose host framework owns every allocation.  This call
 * computes exactly what bl_forward computes, with the same kernels, but keeps
 * the tensor-core path's scratch (int8 activation codes, per-token scales and
 * row sums) in one static device array of the library instead of a caller
 * workspace.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Limits: M*K <= 16 MiB (the int8 codes) and M <= 8192 on the tensor-core path
 * (M > 2); larger shapes return BL_ERR_SCRATCH_LIMIT before anything runs.
 * The decode path (M <= 2) needs no scratch and has no such limit.  The array
 * (16 MiB + 64 KiB) exists on every GPU that loads the library, until the
 * process exits.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  Every call on a device shares the one array: calls whose
 * kernels overlap on the GPU (different streams, or several host threads) race
 * on it and must be serialised by the caller.  Nothing in the array needs to
 * start at zero: every byte a call reads is first written by the same call.
 * Arguments, layouts and status codes are otherwise those of bl_forward.
 */
BL_API bl_status bl_forward_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp,
                                    const float* gamma, int bits, uint16_t* Y, cudaStream_t stream);

/*
 * Grouped forward: up to 8 independent BitLinear problems in one call, e.g.
 * the up, gate and down projections of a feed-forward block at one decode
 * step, or several requests' layers.  Each problem is exactly one bl_forward
 * (same formulas, same rounding, bit-identical results).  When every problem
 * has M == 1 and K <= 8192, all of them share one decode kernel launch,
 * whatever their K (the launch's CTAs are shared out by an estimate of each
 * problem's work), so the fixed cost of a launch is paid once per call;
 * otherwise the problems run one after another on the stream.  The problems
 * are independent: no problem's X may be another problem's Y.  The ordering
 * rule of bl_forward applies to every Wp and gamma.
 * workspace: >= bl_forward_grouped_workspace_bytes(count, problems, bits)
 * (the largest per-problem bl_forward workspace; 0 for an all-decode group).
 * count > 8 returns BL_ERR_UNSUPPORTED; problems with M == 0 are skipped.
 * All problems are validated before anything is launched.
 */
typedef struct {
  const uint16_t* X; /* bf16 bits [M, K], 16-byte aligned */
  int64_t M, K, N;
  const uint8_t* Wp;  /* packed weights [N, K/4], 16-byte aligned */
  const float* gamma; /* device fp32 */
  uint16_t* Y;        /* bf16 bits [M, N] */
} bl_linear;

BL_API size_t bl_forward_grouped_workspace_bytes(int count, const bl_linear* problems, int bits);
BL_API bl_status bl_forward_grouped(int count, const bl_linear* problems, int bits, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream);


/*
 * bl_forward_grouped end to end on host-resident activations: problems[i].X
 * and problems[i].Y are HOST pointers (pinned memory keeps the copies
 * asynchronous); Wp and gamma are device pointers as usual; every problem
 * has at least one token, and no output may overlap an input or another
 * output (BL_ERR_INVALID_ARG).  On `stream`, in order: the inputs copied to
 * the device (problems with the same X, M and K share one copy; inputs whose
 * host bytes are exactly contiguous travel in one copy), the grouped forward
 * of bl_forward_grouped on the staged tensors, the outputs copied back
 * (exactly contiguous outputs in one copy).  A copy of at most 1 MiB is a
 * small kernel that reads or writes the host bytes directly when they are
 * pinned memory the device can address (16-byte aligned); other copies are
 * copy-engine transfers.  Only
 * the tensors' own bytes are read or written.  The call
 * returns once everything is enqueued; the host buffers must stay valid
 * until the stream reaches that point.
 * staging: device memory of at least
 * bl_forward_grouped_host_staging_bytes(count, problems) bytes, 16-byte
 * aligned, owned by the caller (the staged inputs and outputs, 256-byte
 * aligned inside it).  workspace: as bl_forward_grouped (its size query
 * takes the same structs).  Errors: as bl_forward_grouped, plus
 * BL_ERR_WORKSPACE for missing or short staging; nothing is copied or
 * launched unless the whole group is valid.
 */
BL_API size_t bl_forward_grouped_host_staging_bytes(int count, const bl_linear* problems);
BL_API bl_status bl_forward_grouped_host(int count, const bl_linear* problems, int bits, void* staging,
                                         size_t staging_bytes, void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream);
/*
 * The host-buffer grouped forward above, recorded once as a CUDA graph and
 * replayed.  No counterpart on the pages: it serves callers that run the
 * same step over and over on fixed buffers (a serving loop that writes each
 * new token into the same pinned host buffer), for whom the host work of a
 * call -- argument checks, the launch table, one API call per copy and per
 * kernel -- costs several times the GPU time of a one-token step; a replay
 * is one graph launch.
 * bl_forward_grouped_host_graph takes the arguments of
 * bl_forward_grouped_host and keeps their pointers: every replay copies the
 * CURRENT contents of the same host inputs in, runs the same forward and
 * copies the outputs back to the same host outputs, using the same staging,
 * workspace and weights, which must all stay valid (and keep their sizes)
 * until bl_graph_destroy.  Creating it runs the step once on `stream`
 * (the outputs are written) and waits for it, then records the step on a
 * private stream; it must not be called while the calling thread captures
 * a stream.  Errors: as
 * bl_forward_grouped_host (count must be 1..8), plus BL_ERR_CUDA when the
 * capture fails; on error *graph is NULL.
 * bl_graph_launch enqueues one replay on `stream` (asynchronous; replays
 * that overlap on the GPU share the staging and workspace and race).
 * bl_graph_destroy frees the recorded graph (NULL is ignored); no replay may
 * still be running.
 */
typedef struct bl_graph_s* bl_graph;
BL_API bl_status bl_forward_grouped_host_graph(int count, const bl_linear* problems, int bits, void* staging,
                                               size_t staging_bytes, void* workspace, size_t workspace_bytes,
                                               cudaStream_t stream, bl_graph* graph);
BL_API bl_status bl_graph_launch(bl_graph graph, cudaStream_t stream);
BL_API void bl_graph_destroy(bl_graph graph);
/*
 * Squared-ReLU feed-forward: the down projection's input is formed from the
 * gate projection's output ("BitNet 2B4T Guide: Scaling Native 1.58-Bit
 * LLMs", section "2. Squared ReLU Activation", ReLU^2(x) = max(0, x)^2, and
 * the page's feed-forward module, which feeds ReLU^2 of the gate projection
 * to the down projection) and quantised in the same kernel:
 *   h[m,k] = f32( max(0, G[m,k])^2 )                    (U == NULL)
 *   h[m,k] = f32( f32(max(0, G[m,k])^2) * U[m,k] )      (gated, U != NULL)
 * (exact for bf16 G and U), then exactly the per-token quantisation of
 * bl_quant_act applied to the fp32 h, and the rest of bl_forward.
 * G, U: bf16 bits [M, K], 16-byte aligned (U may be NULL).  Wp, gamma, Y and
 * the workspace as in bl_forward (workspace: bl_forward_relu2_workspace_bytes,
 * 0 when M == 1 and K <= 8192: the decode kernel forms h in its prologue).
 * The ordering rule of bl_forward applies; G and U may be written by the
 * preceding kernel of the stream (they are read after the dependency wait).
 */
BL_API size_t bl_forward_relu2_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);
BL_API bl_status bl_forward_relu2(const uint16_t* G, const uint16_t* U, int64_t M, int64_t K, int64_t N,
                                  const uint8_t* Wp, const float* gamma, int bits, uint16_t* Y, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);
/* Test export: the quantisation step of bl_forward_relu2 alone (codes int8
 * [M, K] and scales fp32 [M], as bl_quant_act). */
BL_API bl_status bl_quant_act_relu2(const uint16_t* G, const uint16_t* U, int64_t M, int64_t K, int bits, int8_t* Xq,
                                    float* scale, cudaStream_t stream);


/*
 * The variants the pages print, as one entry point:
 *   BL_ACT_PER_TENSOR  one absmax over the whole activation tensor instead of
 *                      one per token ("BitNet 2B4T Guide: Scaling Native
 *                      1.58-Bit LLMs", section "1. The BitLinear Operator"):
 *                      a = max over all |X|, s = Q / max(a, 1e-5) for every
 *                      row, q = clamp(round_half_even(X * s), -Q-1, Q);
 *   bias               optional fp32 [N] added after the rescale (the
 *                      BitLinear module's bias argument, "BitNet b1.58: The
 *                      1-Bit Ternary LLM Architecture Guide"):
 *                      Y = bf16( f32( f32(f32(acc) * f32(gamma / s_m)) + bias[n] ) ).
 * Otherwise exactly bl_forward.  flags: 0 or BL_ACT_PER_TENSOR (other bits
 * return BL_ERR_UNSUPPORTED); bias may be NULL (4-byte aligned otherwise).
 * workspace: bl_forward_ex_workspace_bytes (0 when M == 1 and K <= 8192).
 * With M > 1 the tensor-core path runs for every M (the per-tensor absmax is
 * one more kernel before the quantiser).
 */
#define BL_ACT_PER_TENSOR 1u
BL_API size_t bl_forward_ex_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits, unsigned flags);
BL_API bl_status bl_forward_ex(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp,
                               const float* gamma, int bits, unsigned flags, const float* bias, uint16_t* Y,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * RMSNorm ahead of the quantisation (SubLN: "BitNet 2B4T Guide: Scaling
 * Native 1.58-Bit LLMs", section "3. Sub-Layer Normalization (SubLN)" and the
 * page's pipeline figure, x_norm = RMSNorm(x) right before the absmax step;
 * the norm's weight kept in bf16 per "BitNet a4.8 Guide: 4-Bit Activation
 * 1-Bit LLMs", table "Best Practices for Deploying BitNet a4.8 in
 * Production", row "LayerNorm Preservation").  Per token m:
 *   ms_m   = fp32_rn( (1/K) sum_k X[m,k]^2 )      the sum exact, one rounding
 *   r_m    = sqrt_rn( f32(ms_m + eps) )
 *   Xn[m,k]= bf16_rn( f32( f32(X[m,k] / r_m) * w[k] ) )   (w == NULL: no product)
 * then exactly bl_forward on Xn (per-token absmax, codes, ternary matmul,
 * rescale).  The result is bit-identical to normalising into a bf16 tensor
 * with these roundings and calling bl_forward on it; nothing is written
 * between the steps except the int8 codes (M > 1).
 * X: bf16 bits [M, K], 16-byte aligned.  norm_weight: bf16 bits [K] or NULL
 * (16-byte aligned).  eps: positive and finite (else BL_ERR_INVALID_ARG).
 * Wp, gamma, Y as in bl_forward.  workspace: at least
 * bl_forward_rmsnorm_workspace_bytes(M, K, N, bits) bytes, 16-byte aligned,
 * required for every M (one token whose layer fits the resident decode kernel
 * forms everything in that kernel's prologue and leaves it untouched; other
 * shapes write the codes and scales there and run the tensor-core GEMM).
 * The ordering rule of bl_forward applies, and norm_weight counts as a
 * parameter like Wp: one-token launches may read it before the dependency
 * wait.  X may be written by the preceding kernel.
 */
BL_API size_t bl_forward_rmsnorm_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);
BL_API bl_status bl_forward_rmsnorm(const uint16_t* X, const uint16_t* norm_weight, float eps, int64_t M, int64_t K,
                                    int64_t N, const uint8_t* Wp, const float* gamma, int bits, uint16_t* Y,
                                    void* workspace, size_t workspace_bytes, cudaStream_t stream);
/* Test export: the normalisation and quantisation step of bl_forward_rmsnorm
 * alone: codes int8 [M, K] and scales fp32 [M] as bl_quant_act, and, when
 * mean_sq is not NULL (4-byte aligned), ms_m fp32 [M]. */
BL_API bl_status bl_quant_act_rmsnorm(const uint16_t* X, const uint16_t* norm_weight, float eps, int64_t M,
                                      int64_t K, int bits, int8_t* Xq, float* scale, float* mean_sq,
                                      cudaStream_t stream);

/*
 * LayerNorm ahead of the quantisation, without affine parameters ("BitNet
 * b1.58: The 1-Bit Ternary LLM Architecture Guide", BitLinear code listing,
 * forward step 1: a layer_norm over the feature axis before the activation
 * quantiser; the "BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs" BitLinear
 * module, a LayerNorm with its affine parameters off).  Per token m:
 *   mu_m   = fp32_rn( (1/K) sum_k X[m,k] )              the sum exact
 *   var_m  = fp32_rn( (1/K) sum_k (X[m,k] - (1/K) sum_j X[m,j])^2 )
 *            the biased variance, exact, one rounding
 *   r_m    = sqrt_rn( f32(var_m + eps) )
 *   Xn[m,k]= bf16_rn( f32( f32(X[m,k] - mu_m) / r_m ) )
 * then exactly bl_forward on Xn.  Arguments, workspace
 * (bl_forward_layernorm_workspace_bytes), errors and ordering as in
 * bl_forward_rmsnorm (there is no weight).
 */
BL_API size_t bl_forward_layernorm_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);
BL_API bl_status bl_forward_layernorm(const uint16_t* X, float eps, int64_t M, int64_t K, int64_t N,
                                      const uint8_t* Wp, const float* gamma, int bits, uint16_t* Y, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream);
/* Test export: the normalisation and quantisation step of bl_forward_layernorm
 * alone: codes and scales as bl_quant_act and, when not NULL (4-byte
 * aligned), mu_m and var_m fp32 [M]. */
BL_API bl_status bl_quant_act_layernorm(const uint16_t* X, float eps, int64_t M, int64_t K, int bits, int8_t* Xq,
                                        float* scale, float* mean, float* var, cudaStream_t stream);

/*
 * Several normalised BitLinear forwards in one call: each problem i is
 * bl_forward_rmsnorm (norm == BL_NORM_RMS, weight norm_weights[i], which may
 * be NULL, or norm_weights == NULL for none) or bl_forward_layernorm (norm ==
 * BL_NORM_LAYER, norm_weights must be NULL) of its own X, with one eps.
 * When every non-empty problem has one token, K <= 8192, and all weights fit
 * the resident decode kernel's rings (sum N*K/4 <= SMs * 96 KiB), the whole
 * group is ONE launch in which every CTA normalises its own problem's token;
 * otherwise the problems run one after another.  At most 8 problems; no
 * problem's X may be another's Y.  workspace: at least
 * bl_forward_norm_grouped_workspace_bytes(count, problems, bits) bytes,
 * 16-byte aligned, reused by the problems in stream order.  Errors as in
 * bl_forward_rmsnorm; BL_ERR_UNSUPPORTED for another norm or more than 8
 * problems.  Nothing is launched unless every problem is valid.
 */
#define BL_NORM_RMS 0
#define BL_NORM_LAYER 1
BL_API size_t bl_forward_norm_grouped_workspace_bytes(int count, const bl_linear* problems, int bits);
BL_API bl_status bl_forward_norm_grouped(int count, const bl_linear* problems, int norm,
                                         const uint16_t* const* norm_weights, float eps, int bits, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream);

/* Device workspace bytes bl_matmul_i32 needs (0 when M <= 2). */
BL_API size_t bl_matmul_i32_workspace_bytes(int64_t M, int64_t K, int64_t N);

/*
 * [b1.58] eq. (3) without the rescale: acc[m,n] = sum_k Xq[m,k] * code[n,k]
 * as exact int32, on already-quantised int8 activations Xq [M, K] (16-byte
 * aligned).  acc: int32 [M, N].  Same kernels as bl_forward.  For tests.
 */
BL_API bl_status bl_matmul_i32(const int8_t* Xq, int64_t M, int64_t K, int64_t N, const uint8_t* Wp, int32_t* acc,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Base-3 weight storage: five ternary weights per byte, 1.6 bits a weight
 * ("BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "Why 1.58
 * Bits? The Power of Zero": a ternary weight carries log2(3) ~ 1.58 bits, and
 * 3^5 = 243 states fit in one byte), i.e. 20% fewer weight bytes than the
 * 2-bit storage for the same codes.  Layout (this library's): a row of K
 * weights is 4 * ceil(ceil(K / 20) / 4) bytes (16-byte multiple) of
 * little-endian 32-bit words; byte b of word g holds the digits
 * d_L = code + 1 of the weights k = 20g + 4L + b (L = 0..4; digits past the
 * end of the row are 1) as ceil(256 * v / 243) with v = sum_L d_L * 3^(4-L).
 * The codes and gamma are exactly those of bl_quantize_weights.
 * ------------------------------------------------------------------------- */

/* N * 4 * ceil(ceil(K / 20) / 4) (0 for an invalid shape). */
BL_API size_t bl_packed_weight_bytes_b3(int64_t N, int64_t K);

/* [b1.58] eq. (1) as bl_quantize_weights, stored in base 3.  Wp3:
 * bl_packed_weight_bytes_b3(N, K) bytes, 16-byte aligned; workspace as for
 * bl_quantize_weights (bl_quantize_weights_workspace_bytes). */
BL_API bl_status bl_quantize_weights_b3(const float* W, int64_t N, int64_t K, uint8_t* Wp3, float* gamma,
                                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Base-3 weights -> int8 codes [N, K].  For tests and inspection. */
BL_API bl_status bl_unpack_weights_b3(const uint8_t* Wp3, int64_t N, int64_t K, int8_t* codes, cudaStream_t stream);

/* bl_forward on base-3 weights, for one token (M == 1, K <= 8192; other
 * shapes return BL_ERR_UNSUPPORTED, M == 0 is a no-op): the same formulas and
 * roundings, so Y is bit-identical to bl_forward on the 2-bit storage of the
 * same codes.  The decode kernel decodes five weights a byte.  No workspace.
 * The ordering rule of bl_forward applies to Wp3 and gamma. */
BL_API bl_status bl_forward_b3(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* Wp3,
                               const float* gamma, int bits, uint16_t* Y, cudaStream_t stream);

/* [b1.58] eq. (3) without the rescale on base-3 weights and int8 codes Xq
 * (M == 1): exact int32 acc [N].  For tests. */
BL_API bl_status bl_matmul_i32_b3(const int8_t* Xq, int64_t M, int64_t K, int64_t N, const uint8_t* Wp3,
                                  int32_t* acc, cudaStream_t stream);

/*
 * Throughput probe of the tensor-core instruction the prefill GEMMs run on
 * (tcgen05.mma kind::i8, A in tensor memory, B in shared memory).  No
 * counterpart on the pages: it measures the peak that the GEMMs' tensor-pipe
 * fraction is quoted against.  grid CTAs (one per SM when grid <= the SM
 * count) each issue n_mma MMAs of M = 128, N = n_cols, K = 32 into one
 * accumulator and write, to out[2*i] and out[2*i+1] (device, 2*grid values),
 * the SM clock cycles and nanoseconds the issue-to-completion took (0 and 0 if
 * the bounded wait gave up).  Rate per SM = 128 * n_cols * 32 * n_mma / cycles
 * multiply-accumulates per clock.  n_mma in [1, 2^22], n_cols a multiple of
 * 16 in [16, 256], grid in [1, 4096] (else BL_ERR_SHAPE).
 */
BL_API bl_status bl_probe_mma_i8(int n_mma, int n_cols, unsigned long long* out, int grid, cudaStream_t stream);
/* The CTA-pair form of the probe (tcgen05.mma cta_group::2, clusters of two
 * CTAs, M = 256 over the pair, N = n_cols with half of B in each CTA): the
 * pair's leader issues the MMAs; every CTA writes its cycles and nanoseconds
 * as above.  Rate per SM = 128 * n_cols * 32 * n_mma / cycles.  grid even,
 * n_cols a multiple of 32 in [32, 256] (else BL_ERR_SHAPE). */
BL_API bl_status bl_probe_mma_i8_pair(int n_mma, int n_cols, unsigned long long* out, int grid, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Device status.
 * ------------------------------------------------------------------------- */

/* Synchronises the current device, then returns the status recorded by
 * kernels since the last clear (BL_OK if none) and, if clear != 0, resets it.
 * If site != NULL it receives the identifier of the wait that gave up. */
BL_API bl_status bl_device_status(int clear, int* site);

/* Launches a one-thread kernel that waits, with the library's bounded wait,
 * on a barrier nothing ever completes; after limit_ns nanoseconds the wait
 * gives up and records BL_ERR_TIMEOUT in the device status word.  *waited_ok
 * (device int) receives 0.  For tests of the failure path. */
BL_API bl_status bl_selftest_wait_timeout(unsigned long long limit_ns, int* waited_ok, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
