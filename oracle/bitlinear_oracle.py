"""CPU oracle for the BitNet b1.58 BitLinear forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: it exists so that tests, the smoke check and the CPU
baseline leg of the benchmark can check the CUDA library against a plain,
slow, obviously correct restatement of what the pages compute.  It shares no
code, constant table or helper with the CUDA library.

Sources (web pages, cited by title and section):

  [P2] "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide",
       section "The Mathematical Formulation of BitLinear":
         eq. (1) absmean weight scale gamma and the ternary round-clip,
         eq. (2) per-token absmax activation scale and round-clip,
         eq. (3) integer matmul followed by one rescale by gamma / scale_X;
       section "Why 1.58 Bits? The Power of Zero": a ternary weight adds,
         subtracts or skips the activation.
  [P1] "BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs",
       section "1. Hybrid W1.58 / A4 Quantization Function": 4-bit
         activation codes clipped to [-8, 7], scale max|X| / 7.
  [P3] "BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs",
       section "1. The BitLinear Operator": clip range [-128, 127] for the
         8-bit codes; the dequantisation factor beta / gamma;
       section "2. Squared ReLU Activation": ReLU^2(x) = (max(0, x))^2
         between the feed-forward projections (the page's module applies it
         to the gate projection's output and feeds the result to the down
         projection);
       section "3. Sub-Layer Normalization (SubLN)" and the pipeline figure
         of the same page: the activations pass through RMSNorm right
         before the absmax quantisation.

Readings where the pages are silent or disagree (each one is listed with its
reason in the design notes of the repository):

  * gamma is the mean of |W| over the whole tensor, computed exactly and
    rounded once to fp32 (round to nearest, ties to even); epsilon enters as
    a floor, gamma = max(mean|W|, 1e-5), and that floored value is both the
    divisor of W and the stored scale.
  * Round() is round-half-to-even everywhere (torch.round semantics).
  * Weight codes: clip(rint(W / gamma), -1, 1), with an IEEE fp32 division.
    Clip-then-round and round-then-clip give the same codes (tested).
  * Activations are quantised per token (per row of X):
        a_m = max_k |x_mk|              (exact; bf16 -> fp32 is exact)
        s_m = Q / max(a_m, 1e-5)        (fp32 division)
        q   = clip(rint(x * s_m), -Q-1, Q)   (fp32 product)
    with Q = 127 (8-bit) or Q = 7 (4-bit a4.8 mode).  The a4.8 page divides
    by max|X|/7 instead of multiplying by 7/max|X|; the multiply form is
    used for both widths (the page's divide form is available as
    ``act_quant(..., a4_divide_form=True)`` so tests can count differences).
  * Rescale: f_m = gamma / s_m and y = acc * f_m.  ``rescale`` returns the
    fp64 value of acc * (gamma / s_m) computed from the fp32 gamma and s_m,
    and the fp32 value obtained with the pages' fp32 tensor arithmetic
    (f32(f32(acc) * f32(gamma / s_m))).  The bf16 output is the
    round-to-nearest-even bf16 of a value.

  * RMSNorm (named, not defined, by the pages): ms = mean of the squares,
    summed exactly and rounded once to fp32; r = sqrt(f32(ms + eps)); the
    normalised value is bf16(f32(f32(x / r) * w)), every step an IEEE fp32
    operation; the weight w (bf16 [K]) is optional.
  * LayerNorm (the code listings' non-affine layer_norm over the feature
    axis, whose eps the pages leave at the library default 1e-5):
    mu = mean of x, the sum exact and rounded once to fp32; var = the
    biased (1/K) variance of x, exact and rounded once; r = sqrt(f32(var +
    eps)); the normalised value is bf16(f32(f32(x - mu) / r)).

Array conventions: X is [M, K] (tokens x in-features) given as raw bf16 bit
patterns (uint16); W is [N, K] fp32 (out-features x in-features, the
nn.Linear convention); Y is [M, N].
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "EPS",
    "QMAX",
    "bf16_bits_to_f32",
    "round_rational_to_f32",
    "round_to_bf16_bits",
    "exact_abs_sum",
    "absmean_scale",
    "ternary_codes",
    "pack_ternary",
    "unpack_ternary",
    "base3_row_bytes",
    "pack_base3",
    "unpack_base3",
    "act_quant",
    "act_quant_values",
    "act_quant_per_tensor",
    "pack_int4",
    "unpack_int4",
    "relu2_input",
    "matmul_i32",
    "rescale",
    "forward",
    "forward_relu2",
    "forward_ex",
    "exact_square_sum",
    "rms_norm",
    "forward_rmsnorm",
    "exact_sum",
    "layer_norm",
    "forward_layernorm",
]

# Floor used for both scales (pages' code listings clamp(min=1e-5)).
EPS = np.float32(1e-5)

# Largest positive code per activation width: Q_b = 2^(b-1) - 1.
QMAX = {8: 127, 4: 7}


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values.  bf16 is the upper half of an fp32,
    so the conversion is exact."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_rational_to_f32(p: int, q: int) -> np.float32:
    """Round the non-negative rational p/q to the nearest fp32, ties to even.

    Plain integer arithmetic: find the binade [2^e, 2^(e+1)) holding p/q,
    form the 24-bit significand by integer division and round on the
    remainder.  Values below the normal range are rounded on the subnormal
    grid 2^-149.
    """
    if p < 0 or q <= 0:
        raise ValueError("round_rational_to_f32 expects p >= 0, q > 0")
    if p == 0:
        return np.float32(0.0)
    e = p.bit_length() - q.bit_length()
    # make 2^e <= p/q < 2^(e+1)
    if (p << max(0, -e)) < (q << max(0, e)):
        e -= 1
    if e < -126:
        # subnormal grid: significand counts units of 2^-149
        shift = 149
    else:
        shift = 23 - e
    if shift >= 0:
        num, den = p << shift, q
    else:
        num, den = p, q << (-shift)
    m, r = divmod(num, den)
    if 2 * r > den or (2 * r == den and (m & 1)):
        m += 1
    # m * 2^-shift is the rounded value; a carry into the next binade
    # (m == 2^24) is still exactly representable.  A rounded value of 2^128
    # or more overflows to infinity (IEEE round to nearest).
    if e > 127 or (e == 127 and m >= (1 << 24)):
        return np.float32(np.inf)
    val = float(m) * 2.0 ** (-shift)   # exact in fp64: m < 2^25
    out = np.float32(val)
    assert float(out) == val, "rounded value must be exactly representable"
    return out


def round_to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """Round real values (fp32 or fp64 arrays) to bf16, nearest-even.

    bf16 keeps 8 significant bits and the fp32 exponent range.  Writing
    |y| = m * 2^e with m in [0.5, 1), the rounded magnitude is
    rint(m * 2^8) * 2^(e-8), and rint rounds half to even.  Below the
    smallest normal bf16 (2^-126) the grid stays at 2^-133.  The result is
    returned as bf16 bit patterns (uint16).
    """
    y64 = np.asarray(y, dtype=np.float64)
    mag = np.abs(y64)
    _, e = np.frexp(mag)
    e = np.maximum(e, -125)
    r = np.rint(np.ldexp(mag, 8 - e))
    val = np.copysign(np.ldexp(r, e - 8), y64)
    with np.errstate(over="ignore"):
        f32 = val.astype(np.float32)
    bits = f32.view(np.uint32)
    finite = np.isfinite(f32)
    assert np.all((bits[finite] & np.uint32(0xFFFF)) == 0)
    return (bits >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# [P2] eq. (1): absmean weight scale and ternary codes
# ---------------------------------------------------------------------------

def exact_abs_sum(W: np.ndarray, chunk: int = 1 << 24) -> int:
    """Exact value of sum_ij |W_ij| as an integer count of 2^-149.

    Every finite fp32 is an integer multiple of 2^-149: a normal value with
    biased exponent e and fraction f is (2^23 + f) * 2^(e-1) units, a
    subnormal is f units.  Units are grouped by exponent; within a group the
    significands are summed exactly (split into 12-bit halves so that every
    float64 partial sum inside np.bincount stays an integer below 2^53), and
    the groups are combined with Python integers.  The tensor is walked in
    chunks only to bound host memory; integer addition makes the order
    irrelevant.
    """
    a_all = np.ascontiguousarray(W, dtype=np.float32).ravel()
    if a_all.size >= (1 << 40):
        raise ValueError("tensor too large for the exact sum")
    total = 0
    for start in range(0, a_all.size, chunk):
        bits = np.abs(a_all[start:start + chunk]).view(np.uint32)
        e = (bits >> np.uint32(23)).astype(np.int64)
        f = (bits & np.uint32(0x7FFFFF)).astype(np.int64)
        if np.any(e == 255):
            raise ValueError("non-finite weight")
        sig = np.where(e > 0, f | (1 << 23), f)
        sh = np.where(e > 0, e - 1, 0)          # value = sig * 2^sh units
        s_hi = np.bincount(sh, weights=(sig >> 12).astype(np.float64), minlength=254)
        s_lo = np.bincount(sh, weights=(sig & 0xFFF).astype(np.float64), minlength=254)
        for k in range(len(s_hi)):
            if s_hi[k] or s_lo[k]:
                total += ((int(s_hi[k]) << 12) + int(s_lo[k])) << k
    return total


def absmean_scale(W: np.ndarray) -> np.float32:
    """gamma = max( fp32( (1/nm) * sum_ij |W_ij| ), 1e-5 ).

    [P2] eq. (1) defines gamma as the mean absolute weight; [P1] calls the
    same quantity beta.  The mean is formed exactly and rounded once.
    """
    n = int(np.asarray(W).size)
    if n == 0:
        raise ValueError("empty weight tensor")
    mean = round_rational_to_f32(exact_abs_sum(W), n << 149)
    return np.float32(max(mean, EPS))


def ternary_codes(W: np.ndarray, gamma: np.float32) -> np.ndarray:
    """[P2] eq. (1): codes = Round(Clip(W / gamma, -1, 1)) in {-1, 0, +1}.

    fp32 division, round half to even, clip to [-1, 1].  Returned as int8.
    """
    w = np.ascontiguousarray(W, dtype=np.float32)
    r = np.rint(w / np.float32(gamma))
    return np.clip(r, -1, 1).astype(np.int8)


# ---------------------------------------------------------------------------
# 2-bit storage.  The pages fix only the size (2 bits per weight, the
# verification harness of [P1] Step 4 counts in*out*2/8 bytes); the layout
# below is this library's format.
#
#   * byte offset of row n is n*K/4; rows are K/4 bytes.
#   * the row is a sequence of little-endian 32-bit words; word g holds the
#     16 weights k = 16g .. 16g+15.
#   * weight k = 16g + 4j + b (j, b in 0..3) sits in bits [8b+2j, 8b+2j+2)
#     of word g.
#   * the 2-bit field holds u = code + 1: 0 -> -1, 1 -> 0, 2 -> +1
#     (3 is never written).
# ---------------------------------------------------------------------------

def pack_ternary(codes: np.ndarray) -> np.ndarray:
    """int8 codes [N, K] (K % 16 == 0) -> packed uint8 [N, K/4]."""
    c = np.asarray(codes)
    N, K = c.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    u = (c.astype(np.int64) + 1).reshape(N, K // 16, 4, 4)   # [n, g, j, b]
    if np.any((u < 0) | (u > 2)):
        raise ValueError("codes must lie in {-1, 0, 1}")
    words = np.zeros((N, K // 16), dtype=np.uint64)
    for j in range(4):
        for b in range(4):
            words |= u[:, :, j, b].astype(np.uint64) << np.uint64(8 * b + 2 * j)
    return words.astype("<u4").view(np.uint8).reshape(N, K // 4)


def unpack_ternary(packed: np.ndarray, K: int) -> np.ndarray:
    """packed uint8 [N, K/4] -> int8 codes [N, K] (inverse of pack_ternary)."""
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    N = p.shape[0]
    words = p.reshape(N, K // 4).view("<u4").astype(np.uint64)   # [N, K/16]
    out = np.empty((N, K // 16, 4, 4), dtype=np.int64)
    for j in range(4):
        for b in range(4):
            out[:, :, j, b] = (words >> np.uint64(8 * b + 2 * j)) & np.uint64(3)
    if np.any(out == 3):
        raise ValueError("reserved 2-bit value 3 found")
    return (out.reshape(N, K) - 1).astype(np.int8)


# ---------------------------------------------------------------------------
# Base-3 storage: five ternary weights per byte ([P2] section "Why 1.58 Bits?
# The Power of Zero": three states carry log2(3) ~ 1.58 bits; 3^5 = 243 states
# fit in one byte, 1.6 bits a weight).  The pages fix only the density; the
# layout is this library's:
#   * a row of K weights is a run of little-endian 32-bit words padded to a
#     multiple of four words (16 bytes); word g holds k = 20g .. 20g+19;
#   * byte b (0..3) of word g holds the five digits d_L = code + 1 (L = 0..4)
#     of the weights k = 20g + 4L + b; digits past the end of the row are 1
#     (code 0);
#   * the byte stores ceil(256 * v / 243) with v = sum_L d_L * 3^(4 - L), the
#     base-3 number whose most significant digit is d_0.  (v is recovered
#     exactly as floor(243 * byte / 256); the scaled form lets a decoder get
#     the digits in order by repeated multiplication by 3.)
# ---------------------------------------------------------------------------

def base3_row_bytes(K: int) -> int:
    """Bytes of one base-3 row of K weights (16-byte multiple)."""
    words = -(-K // 20)
    return 4 * (-(-words // 4) * 4)


def pack_base3(codes: np.ndarray) -> np.ndarray:
    """int8 codes [N, K] in {-1, 0, 1} -> base-3 bytes [N, base3_row_bytes(K)]."""
    c = np.asarray(codes)
    N, K = c.shape
    d = c.astype(np.int64) + 1
    if np.any((d < 0) | (d > 2)):
        raise ValueError("codes must lie in {-1, 0, 1}")
    rb = base3_row_bytes(K)
    padded = np.ones((N, rb * 5), dtype=np.int64)        # digit 1 = code 0
    padded[:, :K] = d
    # word g, level L, byte b <-> k = 20g + 4L + b
    digits = padded.reshape(N, rb // 4, 5, 4)              # [n, g, L, b]
    v = np.zeros((N, rb // 4, 4), dtype=np.int64)
    for L in range(5):
        v += digits[:, :, L, :] * 3 ** (4 - L)
    q = -((-256 * v) // 243)                               # ceil(256 v / 243)
    return q.reshape(N, rb).astype(np.uint8)


def unpack_base3(packed: np.ndarray, K: int) -> np.ndarray:
    """Base-3 bytes [N, base3_row_bytes(K)] -> int8 codes [N, K] (inverse of
    pack_base3: v = floor(243 * byte / 256), then its base-3 digits)."""
    p = np.ascontiguousarray(packed, dtype=np.uint8).astype(np.int64)
    N, rb = p.shape
    if rb != base3_row_bytes(K):
        raise ValueError("row length does not match K")
    v = (243 * p) // 256
    if np.any(v > 242):
        raise ValueError("byte outside the 243 base-3 states")
    v = v.reshape(N, rb // 4, 4)                           # [n, g, b]
    digits = np.empty((N, rb // 4, 5, 4), dtype=np.int64)
    for L in range(5):
        digits[:, :, L, :] = (v // 3 ** (4 - L)) % 3
    return (digits.reshape(N, rb * 5)[:, :K] - 1).astype(np.int8)


# ---------------------------------------------------------------------------
# [P2] eq. (2) and [P1] section 1: per-token absmax activation quantisation
# ---------------------------------------------------------------------------

def act_quant(x_bits: np.ndarray, bits: int = 8, a4_divide_form: bool = False):
    """Quantise bf16 activations [M, K] per token.

    Returns (q int8 [M, K], s fp32 [M]) with s_m = Q / max(a_m, 1e-5) and
    q = clip(rint(x * s_m), -Q-1, Q).  With ``a4_divide_form`` (4-bit only)
    the codes follow the a4.8 page literally, q = clip(rint(x / (a'/7))),
    and the returned s_m is still Q / a'.
    """
    if bits not in QMAX:
        raise ValueError("bits must be 8 or 4")
    Q = QMAX[bits]
    x = bf16_bits_to_f32(x_bits)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    a = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    a_floor = np.maximum(a, EPS).astype(np.float32)
    s = (np.float32(Q) / a_floor).astype(np.float32)
    if a4_divide_form:
        if bits != 4:
            raise ValueError("the divide form is the 4-bit page's form")
        step = (a_floor / np.float32(7.0)).astype(np.float32)
        t = x / step[:, None]
    else:
        t = x * s[:, None]
    q = np.clip(np.rint(t), -Q - 1, Q).astype(np.int8)
    return q, s


def act_quant_values(x: np.ndarray, bits: int = 8):
    """The same per-token quantisation as ``act_quant`` on fp32 values that
    need not be bf16 (the squared-ReLU feed-forward input):
    s_m = Q / max(max_k |x_mk|, 1e-5), q = clip(rint(f32(x * s_m)), -Q-1, Q).
    Returns (q int8 [M, K], s fp32 [M])."""
    if bits not in QMAX:
        raise ValueError("bits must be 8 or 4")
    Q = QMAX[bits]
    xf = np.asarray(x, dtype=np.float32)
    if xf.ndim != 2:
        raise ValueError("x must be [M, K]")
    a = np.max(np.abs(xf), axis=1) if xf.shape[1] else np.zeros(xf.shape[0], np.float32)
    a_floor = np.maximum(a, EPS).astype(np.float32)
    s = (np.float32(Q) / a_floor).astype(np.float32)
    t = (xf * s[:, None]).astype(np.float32)
    q = np.clip(np.rint(t), -Q - 1, Q).astype(np.int8)
    return q, s


def act_quant_per_tensor(x_bits: np.ndarray, bits: int = 8):
    """The per-tensor variant ([P3] section "1. The BitLinear Operator"
    quantises with one absmax over the whole activation tensor): a = max over
    every |x|, s = Q / max(a, 1e-5) (fp32), q = clip(rint(f32(x * s)), -Q-1, Q).
    Returns (q int8 [M, K], s fp32 [M], every entry the same scale)."""
    if bits not in QMAX:
        raise ValueError("bits must be 8 or 4")
    Q = QMAX[bits]
    x = bf16_bits_to_f32(x_bits)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    a = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    s1 = np.float32(np.float32(Q) / np.maximum(a, EPS))
    t = (x * s1).astype(np.float32)
    q = np.clip(np.rint(t), -Q - 1, Q).astype(np.int8)
    return q, np.full(x.shape[0], s1, dtype=np.float32)


# ---------------------------------------------------------------------------
# [P3] section 2: squared ReLU between the feed-forward projections
# ---------------------------------------------------------------------------

def pack_int4(q: np.ndarray) -> np.ndarray:
    """4-bit activation codes int8 [M, K] in [-8, 7] -> packed uint8 [M, K/2]
    ([P1] "Step 4: Verification and Benchmarking Test Harness" counts the 4-bit
    activations at half a byte each).  The layout is this library's: byte j of
    row m holds code 2j in its low nibble and code 2j + 1 in its high nibble,
    each as a 4-bit two's-complement number."""
    c = np.asarray(q, dtype=np.int64)
    M, K = c.shape
    if K % 2:
        raise ValueError("K must be even")
    if np.any((c < -8) | (c > 7)):
        raise ValueError("codes must lie in [-8, 7]")
    nib = c & 0xF
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray, K: int) -> np.ndarray:
    """Inverse of pack_int4: packed uint8 [M, K/2] -> int8 codes [M, K]."""
    p = np.asarray(packed, dtype=np.int64)
    M = p.shape[0]
    out = np.empty((M, K), dtype=np.int64)
    lo, hi = p & 0xF, (p >> 4) & 0xF
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out.astype(np.int8)


def relu2_input(g_bits: np.ndarray, u_bits: np.ndarray | None = None) -> np.ndarray:
    """Input of the down projection from the gate projection's bf16 output g:
    h = max(0, g)^2 in fp32; with ``u_bits`` (the up projection's output, the
    gated variant) h = f32(max(0, g)^2 * u).  For bf16 g and u both products
    are exact in fp32 (8 + 8 and 16 + 8 significant bits), barring overflow."""
    g = bf16_bits_to_f32(g_bits)
    r = np.maximum(g, np.float32(0.0)).astype(np.float32)
    h = (r * r).astype(np.float32)
    if u_bits is not None:
        h = (h * bf16_bits_to_f32(u_bits)).astype(np.float32)
    return h


# ---------------------------------------------------------------------------
# [P2] eq. (3): integer matmul and rescale
# ---------------------------------------------------------------------------

def matmul_i32(q: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * codes[n, k], exact, as int32.

    The product is taken with a float64 matmul: every product and partial
    sum is an integer of magnitude <= 128 * K < 2^53, so each float64
    operation is exact whatever the summation order.
    """
    qq = np.asarray(q)
    cc = np.asarray(codes)
    K = qq.shape[1]
    if 128 * K >= (1 << 53):
        raise ValueError("K too large for an exact float64 matmul")
    acc = qq.astype(np.float64) @ cc.astype(np.float64).T
    out = acc.astype(np.int64)
    assert np.all(out == acc)
    if np.any(np.abs(out) >= (1 << 31)):
        raise OverflowError("accumulator exceeds int32")
    return out.astype(np.int32)


def rescale(acc: np.ndarray, gamma: np.float32, s: np.ndarray):
    """Y = acc * (gamma / scale_X), per row m.

    Returns (y64, y32):
      y64 = float64(acc) * (float64(gamma) / float64(s_m))
      y32 = f32(f32(acc) * f32(gamma / s_m))   (the pages' fp32 tensors)
    """
    a = np.asarray(acc)
    s32 = np.asarray(s, dtype=np.float32)
    g32 = np.float32(gamma)
    y64 = a.astype(np.float64) * (np.float64(g32) / s32.astype(np.float64))[:, None]
    f32 = (g32 / s32).astype(np.float32)
    y32 = (a.astype(np.float32) * f32[:, None]).astype(np.float32)
    return y64, y32


def forward(x_bits: np.ndarray, W: np.ndarray, bits: int = 8):
    """Whole BitLinear forward on bf16 activations and fp32 latent weights.

    Returns a dict with every intermediate: gamma, codes, packed, q, s, acc,
    y64, y32, and Y (bf16 bits of round-to-nearest-even of y32).
    """
    gamma = absmean_scale(W)
    codes = ternary_codes(W, gamma)
    q, s = act_quant(x_bits, bits)
    acc = matmul_i32(q, codes)
    y64, y32 = rescale(acc, gamma, s)
    return {
        "gamma": gamma,
        "codes": codes,
        "packed": pack_ternary(codes) if codes.shape[1] % 16 == 0 else None,
        "q": q,
        "s": s,
        "acc": acc,
        "y64": y64,
        "y32": y32,
        "Y": round_to_bf16_bits(y32),
    }


def forward_relu2(g_bits: np.ndarray, u_bits: np.ndarray | None, W: np.ndarray, bits: int = 8):
    """Down projection of the squared-ReLU feed-forward block: BitLinear on
    h = relu2_input(g, u).  Same dict as ``forward`` plus h."""
    h = relu2_input(g_bits, u_bits)
    gamma = absmean_scale(W)
    codes = ternary_codes(W, gamma)
    q, s = act_quant_values(h, bits)
    acc = matmul_i32(q, codes)
    y64, y32 = rescale(acc, gamma, s)
    return {
        "h": h,
        "gamma": gamma,
        "codes": codes,
        "q": q,
        "s": s,
        "acc": acc,
        "y64": y64,
        "y32": y32,
        "Y": round_to_bf16_bits(y32),
    }


def forward_ex(x_bits: np.ndarray, W: np.ndarray, bits: int = 8, per_tensor: bool = False,
               bias: np.ndarray | None = None):
    """``forward`` with the two variants the pages print: per-tensor
    activation scale ([P3] section 1) and an output bias added after the
    rescale ([P2] BitLinear module, ``bias`` argument): y32 = f32(f32(f32(acc)
    * f32(gamma / s_m)) + bias_n), y64 = acc * gamma / s_m + bias_n."""
    gamma = absmean_scale(W)
    codes = ternary_codes(W, gamma)
    q, s = act_quant_per_tensor(x_bits, bits) if per_tensor else act_quant(x_bits, bits)
    acc = matmul_i32(q, codes)
    y64, y32 = rescale(acc, gamma, s)
    if bias is not None:
        b = np.asarray(bias, dtype=np.float32)
        y64 = y64 + b.astype(np.float64)[None, :]
        y32 = (y32 + b[None, :]).astype(np.float32)
    return {"gamma": gamma, "codes": codes, "q": q, "s": s, "acc": acc, "y64": y64, "y32": y32,
            "Y": round_to_bf16_bits(y32)}


# ---------------------------------------------------------------------------
# [P3] section "3. Sub-Layer Normalization (SubLN)": RMS normalisation of the
# activations immediately before their absmax quantisation
# ---------------------------------------------------------------------------

def exact_square_sum(x_bits: np.ndarray) -> int:
    """Exact value of sum_k x_k^2 over bf16 values, as an integer count of
    2^-266 (the square of the smallest bf16 subnormal, 2^-133).

    A finite bf16 with biased exponent e and 7-bit fraction f is
    sig * 2^(max(e, 1) - 134) with sig = 128 + f for e > 0 and sig = f for
    e = 0, so its square is sig^2 * 2^(2 max(e, 1) - 2) units.  Squares are
    grouped by exponent (each group's significand sum is an integer below
    2^53, exact in np.bincount's float64) and the groups are combined with
    Python integers.
    """
    b = np.ascontiguousarray(x_bits, dtype=np.uint16).ravel().astype(np.int64)
    e = (b >> 7) & 0xFF
    f = b & 0x7F
    if np.any(e == 255):
        raise ValueError("non-finite activation")
    if b.size >= (1 << 36):
        raise ValueError("too many values for the exact sum")
    sig = np.where(e > 0, f | 0x80, f)
    sh = 2 * np.maximum(e, 1) - 2
    groups = np.bincount(sh, weights=(sig * sig).astype(np.float64), minlength=510)
    total = 0
    for k in range(len(groups)):
        if groups[k]:
            total += int(groups[k]) << k
    return total


def rms_norm(x_bits: np.ndarray, weight_bits: np.ndarray | None = None, eps: float = 1e-5):
    """RMSNorm of bf16 activations [M, K], per token, with an optional bf16
    weight [K] ([P1] best-practice table, row "LayerNorm Preservation": the
    normalisation parameters stay in bf16).

    The pages name the operation (x_norm = RMSNorm(x) ahead of the absmax
    step in [P3]'s pipeline figure) but fix no precision.  Reading:
        ms  = fp32( (1/K) sum_k x_k^2 )      exact sum, rounded once
        r   = sqrt( f32(ms + eps) )          fp32 square root (IEEE)
        t   = f32(x / r)                     fp32 division (IEEE)
        t   = f32(t * w_k)                   only with a weight
        x_n = bf16(t)                        round to nearest even
    x_n is what a bf16 model hands to the BitLinear layer, so the fused
    operation equals ``forward`` applied to x_n.

    Returns a dict: ms fp32 [M], r fp32 [M], xn bf16 bits [M, K].
    """
    x = bf16_bits_to_f32(x_bits)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    if K == 0:
        raise ValueError("K must be positive")
    e32 = np.float32(eps)
    if not (np.isfinite(e32) and e32 > 0):
        raise ValueError("eps must be a positive finite fp32 value")
    ms = np.empty(M, np.float32)
    for m in range(M):
        ms[m] = round_rational_to_f32(exact_square_sum(x_bits[m]), K << 266)
    v = (ms + e32).astype(np.float32)
    r = np.sqrt(v).astype(np.float32)
    t = (x / r[:, None]).astype(np.float32)
    if weight_bits is not None:
        w = bf16_bits_to_f32(weight_bits)
        if w.shape != (K,):
            raise ValueError("weight must be [K]")
        t = (t * w[None, :]).astype(np.float32)
    return {"ms": ms, "r": r, "xn": round_to_bf16_bits(t)}


def forward_rmsnorm(x_bits: np.ndarray, W: np.ndarray, weight_bits: np.ndarray | None = None,
                    eps: float = 1e-5, bits: int = 8):
    """BitLinear on the RMS-normalised activations: ``forward(rms_norm(x))``.
    Same dict as ``forward`` plus ms, r and xn."""
    nrm = rms_norm(x_bits, weight_bits, eps)
    out = forward(nrm["xn"], W, bits)
    out.update(nrm)
    return out


# ---------------------------------------------------------------------------
# [P2] "BitLinear" code listing (forward step 1) and [P3]'s BitLinear module:
# a LayerNorm without affine parameters over the feature axis, immediately
# before the absmax quantisation
# ---------------------------------------------------------------------------

def exact_sum(x_bits: np.ndarray) -> int:
    """Exact value of sum_k x_k over bf16 values, as a signed integer count
    of 2^-133 (the smallest bf16 subnormal).

    x = (-1)^s sig * 2^(max(e, 1) - 1) units, with sig as in
    ``exact_square_sum``; values are grouped by exponent (a group's signed
    significand sum is an integer below 2^53 in magnitude, exact in float64)
    and the groups are combined with Python integers.
    """
    b = np.ascontiguousarray(x_bits, dtype=np.uint16).ravel().astype(np.int64)
    e = (b >> 7) & 0xFF
    f = b & 0x7F
    if np.any(e == 255):
        raise ValueError("non-finite activation")
    if b.size >= (1 << 36):
        raise ValueError("too many values for the exact sum")
    sig = np.where(e > 0, f | 0x80, f)
    sig = np.where((b >> 15) & 1, -sig, sig)
    sh = np.maximum(e, 1) - 1
    groups = np.bincount(sh, weights=sig.astype(np.float64), minlength=254)
    total = 0
    for k in range(len(groups)):
        if groups[k]:
            total += int(groups[k]) << k
    return total


def layer_norm(x_bits: np.ndarray, eps: float = 1e-5):
    """Non-affine LayerNorm of bf16 activations [M, K], per token.

    The listings normalise with the library's layer_norm and no weight or
    bias; the pages fix no precision.  Reading (every rounding named):
        mu  = fp32( (1/K) sum_k x_k )                  exact sum, rounded once
        var = fp32( (1/K) sum_k (x_k - (1/K) sum_j x_j)^2 )
              the biased variance, exact, rounded once
        r   = sqrt( f32(var + eps) )                   fp32 square root (IEEE)
        d   = f32(x - mu)                              fp32 subtraction
        t   = f32(d / r)                               fp32 division (IEEE)
        x_n = bf16(t)                                  round to nearest even
    The exact variance is formed as (K * sum x^2 - (sum x)^2) / K^2 from the
    two exact sums.

    Returns a dict: mean fp32 [M], var fp32 [M], r fp32 [M], t fp32 [M, K],
    xn bf16 bits [M, K].
    """
    x = bf16_bits_to_f32(x_bits)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    if K == 0:
        raise ValueError("K must be positive")
    e32 = np.float32(eps)
    if not (np.isfinite(e32) and e32 > 0):
        raise ValueError("eps must be a positive finite fp32 value")
    mean = np.empty(M, np.float32)
    var = np.empty(M, np.float32)
    for m in range(M):
        s1 = exact_sum(x_bits[m])          # units 2^-133
        s2 = exact_square_sum(x_bits[m])   # units 2^-266
        mu = round_rational_to_f32(abs(s1), K << 133)
        mean[m] = -mu if s1 < 0 else mu
        num = K * s2 - s1 * s1             # K^2 var, units 2^-266; >= 0
        var[m] = round_rational_to_f32(num, (K * K) << 266)
    v = (var + e32).astype(np.float32)
    r = np.sqrt(v).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        d = (x - mean[:, None]).astype(np.float32)
        t = (d / r[:, None]).astype(np.float32)
    return {"mean": mean, "var": var, "r": r, "t": t, "xn": round_to_bf16_bits(t)}


def forward_layernorm(x_bits: np.ndarray, W: np.ndarray, eps: float = 1e-5, bits: int = 8):
    """BitLinear on the layer-normalised activations: ``forward(layer_norm(x))``.
    Same dict as ``forward`` plus mean, var, r and xn."""
    nrm = layer_norm(x_bits, eps)
    out = forward(nrm["xn"], W, bits)
    out.update({k: nrm[k] for k in ("mean", "var", "r", "xn")})
    return out
