"""Pins for the CPU oracle: each test checks it against something other than
itself -- hand-worked values, closed forms, brute force with exact rational
arithmetic, an independent library conversion, or an invariant the pages state.

Sources: "BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide" (P2),
"BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs" (P1),
"BitNet 2B4T Guide: Scaling Native 1.58-Bit LLMs" (P3).
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import bitlinear_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_bits(values):
    return np.asarray(values, dtype=np.float32).view(np.uint32)


def to_bf16_bits_exact(values):
    """bf16 bit patterns of values that are exactly representable in bf16."""
    b = f32_bits(values)
    assert np.all((b & 0xFFFF) == 0), "test value not exactly representable in bf16"
    return (b >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_round_rational_matches_ieee_on_exact_doubles():
    # p/q with q a power of two and p < 2^53 is an exact double, so numpy's
    # double -> float conversion (IEEE round-to-nearest-even) is a single,
    # correct rounding to compare against.
    rng = np.random.default_rng(1)
    for _ in range(3000):
        p = int(rng.integers(1, 1 << 53))
        sh = int(rng.integers(-60, 200))
        if sh >= 0:
            num, den = p, 1 << sh
        else:
            num, den = p << (-sh), 1
        want = np.float32(float(Fraction(num, den)))
        got = o.round_rational_to_f32(num, den)
        assert got == want and np.signbit(got) == np.signbit(want), (num, den)


def test_round_rational_hand_cases():
    # ties to even on integers: spacing of fp32 in [2^24, 2^25) is 2
    assert o.round_rational_to_f32((1 << 24) + 1, 1) == np.float32(1 << 24)
    assert o.round_rational_to_f32((1 << 24) + 3, 1) == np.float32((1 << 24) + 4)
    # well-known fp32 bit patterns of 1/3, 2/3 and 1/10
    assert f32_bits(o.round_rational_to_f32(1, 3)) == 0x3EAAAAAB
    assert f32_bits(o.round_rational_to_f32(2, 3)) == 0x3F2AAAAB
    assert f32_bits(o.round_rational_to_f32(1, 10)) == 0x3DCCCCCD
    # subnormal grid 2^-149: half of the smallest subnormal ties to 0,
    # 1.5 units ties to 2 units
    assert o.round_rational_to_f32(1, 1 << 150) == np.float32(0.0)
    assert f32_bits(o.round_rational_to_f32(3, 1 << 150)) == 2
    assert f32_bits(o.round_rational_to_f32(1, 1 << 149)) == 1
    # carry into the next binade: 2^24 - 1/2 rounds (tie, even) to 2^24
    assert o.round_rational_to_f32((1 << 25) - 1, 2) == np.float32(1 << 24)


def test_bf16_rounding_hand_cases():
    cases = {
        1.0: 0x3F80,
        1.0 + 2.0 ** -8: 0x3F80,            # tie between 1 and 1+2^-7 -> even
        1.0 + 3 * 2.0 ** -8: 0x3F82,        # tie -> 1 + 2^-6 (even)
        1.0 + 3 * 2.0 ** -9: 0x3F81,        # above the tie -> 1 + 2^-7
        -2.5: 0xC020,
        0.9148622047: 0x3F6A,               # 234/256
        0.0: 0x0000,
    }
    for v, bits in cases.items():
        assert int(o.round_to_bf16_bits(np.array([v]))[0]) == bits, v


def test_bf16_rounding_matches_torch():
    # torch's fp32 -> bf16 cast is an independent round-to-nearest-even
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200000).astype(np.float32),
        # exact ties: bf16 value + half an ulp
        (f32_bits(rng.standard_normal(10000).astype(np.float32)) & 0xFFFF0000 | 0x8000).view(np.float32),
    ]).astype(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.round_to_bf16_bits(x)
    assert np.array_equal(got, want)


def test_bf16_bits_to_f32_exact():
    b = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = o.bf16_bits_to_f32(b)
    t = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    fin = np.isfinite(t)
    assert np.array_equal(f[fin], t[fin])


# ---------------------------------------------------------------------------
# [P2] eq. (1): gamma and the ternary codes
# ---------------------------------------------------------------------------

def test_exact_abs_sum_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(20):
        n = int(rng.integers(8, 400))
        mags = rng.integers(-150, 60, n).astype(np.float64)
        w = (rng.standard_normal(n) * 2.0 ** mags).astype(np.float32)
        w[rng.random(n) < 0.1] = 0.0
        if trial % 3 == 0:   # some subnormals
            w[:5] = np.array([1e-45, -3e-45, 1e-40, 2e-39, -1e-38], np.float32)
        want = sum(Fraction(float(abs(v))) for v in w) * (1 << 149)
        assert want.denominator == 1
        assert o.exact_abs_sum(w) == want.numerator
        # chunking must not change the result
        assert o.exact_abs_sum(w, chunk=7) == want.numerator


def test_gamma_is_correctly_rounded_mean():
    # [1, 2^-24, 2^-60, 0]: mean = 1/4 + 2^-26 + 2^-62, just above the
    # midpoint between 0.25 and 0.25 + 2^-25 -> rounds up.  Summing in
    # float64 first loses the 2^-60 and lands exactly on the midpoint
    # (ties-to-even -> 0.25), so this pins the single exact rounding.
    w = np.array([[1.0, 2.0 ** -24, 2.0 ** -60, 0.0]], np.float32)
    assert o.absmean_scale(w) == np.float32(0.25 + 2.0 ** -25)
    naive = np.float32(np.float64(np.abs(w).astype(np.float64).sum()) / 4)
    assert naive == np.float32(0.25)
    # [1, 2^-24, 2^-24, 0]: mean = 0.25 + 2^-25, exactly representable;
    # a sequential fp32 sum gives 0.25
    w = np.array([[1.0, 2.0 ** -24, 2.0 ** -24, 0.0]], np.float32)
    assert o.absmean_scale(w) == np.float32(0.25 + 2.0 ** -25)


def test_gamma_closed_forms():
    # all |W| equal -> gamma is that value
    w = np.full((8, 64), -0.0390625, np.float32)
    w[::2] *= -1
    assert o.absmean_scale(w) == np.float32(0.0390625)
    # dyadic mean: sum |W| = 0.8125 over 4 -> 0.203125
    assert o.absmean_scale(np.array([[0.375, -0.0625, -0.25, 0.125]], np.float32)) == np.float32(0.203125)
    # epsilon floor
    assert o.absmean_scale(np.zeros((3, 16), np.float32)) == o.EPS
    assert o.absmean_scale(np.full((2, 2), 1e-7, np.float32)) == o.EPS
    # a mean of exactly 1e-5f stays 1e-5f
    assert o.absmean_scale(np.full((2, 2), np.float32(1e-5), np.float32)) == o.EPS


def test_gamma_gaussian_matches_fsum():
    # On real data the exact mean and an fp64 sum agree after rounding to
    # fp32 except with probability ~1e-9; a mismatch here means a bug.
    rng = np.random.default_rng(4)
    for std in (0.02, 0.01, 1.0):
        w = (rng.standard_normal((257, 300)) * std).astype(np.float32)
        ref = np.float32(math.fsum(np.abs(w).astype(np.float64).ravel()) / w.size)
        assert o.absmean_scale(w) == ref


def test_ternary_codes_ties_and_clip():
    # W/gamma = [0.5, -0.5, 1.5, -1.5, 0.4, 0.8, -4, 0, 2.5]
    g = np.float32(0.25)
    w = np.array([[0.125, -0.125, 0.375, -0.375, 0.1, 0.2, -1.0, 0.0, 0.625]], np.float32)
    assert o.ternary_codes(w, g).tolist() == [[0, 0, 1, -1, 0, 1, -1, 0, 1]]


def test_clip_round_commute():
    # Round(Clip(v, -1, 1)) (P2 eq. 1) equals Clip(Round(v), -1, 1) (P1, P3)
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.5, -0.5, 1.5, -1.5, 1.0, -1.0, 0.0], np.float32)])
    a = np.rint(np.clip(v, -1, 1))
    b = np.clip(np.rint(v), -1, 1)
    assert np.array_equal(a, b)


def test_gaussian_zero_fraction():
    # For W ~ N(0, s^2), gamma ~ E|W| = s*sqrt(2/pi) and a weight is coded 0
    # when |W| < gamma/2: P = erf(0.5*sqrt(2/pi)/sqrt(2)) = erf(1/(2*sqrt(pi))).
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((1000, 1000)) * 0.02).astype(np.float32)
    c = o.ternary_codes(w, o.absmean_scale(w))
    p0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    assert abs(p0 - 0.3101) < 1e-3
    assert abs(float(np.mean(c == 0)) - p0) < 3e-3
    assert set(np.unique(c).tolist()) <= {-1, 0, 1}
    # symmetric
    assert abs(float(np.mean(c == 1)) - float(np.mean(c == -1))) < 3e-3


# ---------------------------------------------------------------------------
# 2-bit storage (P1 Step 4 byte count; the bit layout is this library's)
# ---------------------------------------------------------------------------

def test_packed_layout_golden():
    g = json.load(open(os.path.join(GOLDEN, "packed_layout.json")))
    K = g["K"]
    codes = np.zeros((1, K), np.int8)
    for k, v in g["nonzero_codes"].items():
        codes[0, int(k)] = v
    packed = o.pack_ternary(codes)
    assert packed.tolist() == [g["packed_bytes"]]
    assert np.array_equal(o.unpack_ternary(packed, K), codes)


def test_pack_roundtrip_and_size():
    rng = np.random.default_rng(7)
    for N, K in [(1, 16), (3, 64), (17, 256), (64, 1024)]:
        c = rng.integers(-1, 2, (N, K)).astype(np.int8)
        p = o.pack_ternary(c)
        assert p.shape == (N, K // 4) and p.nbytes == N * K * 2 // 8
        assert np.array_equal(o.unpack_ternary(p, K), c)
        # field value 3 never written
        w = p.view("<u4")
        for sh in range(0, 32, 2):
            assert not np.any(((w >> sh) & 3) == 3)


def test_unpack_bytewise_definition():
    # decode one random row bit by bit from the layout definition
    rng = np.random.default_rng(8)
    K = 64
    c = rng.integers(-1, 2, (1, K)).astype(np.int8)
    p = o.pack_ternary(c)[0]
    for k in range(K):
        g, r = divmod(k, 16)
        j, b = divmod(r, 4)
        byte = p[4 * g + b]
        assert ((int(byte) >> (2 * j)) & 3) - 1 == c[0, k]


# ---------------------------------------------------------------------------
# Base-3 storage (P2 "Why 1.58 Bits?": 3^5 = 243 states in a byte; the layout
# is this library's)
# ---------------------------------------------------------------------------

def test_base3_layout_golden():
    g = json.load(open(os.path.join(GOLDEN, "base3_layout.json")))
    K = g["K"]
    codes = np.zeros((1, K), np.int8)
    for k, v in g["nonzero_codes"].items():
        codes[0, int(k)] = v
    packed = o.pack_base3(codes)
    assert packed.tolist() == [g["packed_bytes"]]
    assert np.array_equal(o.unpack_base3(packed, K), codes)


def test_base3_every_byte_decodes_by_repeated_tripling():
    # all 243 digit tuples: the stored bytes are distinct, and the digits come
    # back in order from x -> 3x mod 256 (digit = floor(3x / 256)), a decode
    # independent of the oracle's exact inverse floor(243 * byte / 256)
    import itertools
    seen = set()
    for digits in itertools.product(range(3), repeat=5):
        codes = np.zeros((1, 64), np.int8)
        for L, d in enumerate(digits):
            codes[0, 4 * L] = d - 1          # word 0, byte 0, level L
        byte = int(o.pack_base3(codes)[0, 0])
        assert 0 <= byte <= 255 and byte not in seen
        seen.add(byte)
        x = byte
        got = []
        for _ in range(5):
            got.append((3 * x) >> 8)
            x = (3 * x) & 0xFF
        assert tuple(got) == digits, (digits, byte, got)
    assert len(seen) == 243


def test_base3_roundtrip_sizes_and_padding():
    rng = np.random.default_rng(9)
    for N, K in [(1, 64), (3, 192), (5, 2560), (2, 6912), (1, 8192)]:
        c = rng.integers(-1, 2, (N, K)).astype(np.int8)
        p = o.pack_base3(c)
        words = -(-K // 20)
        assert p.shape == (N, 4 * (-(-words // 4) * 4)) and p.shape[1] % 16 == 0
        assert p.shape[1] * 8 <= 1.61 * K + 128          # ~1.6 bits a weight
        assert np.array_equal(o.unpack_base3(p, K), c)
        # the same codes in both storages
        assert np.array_equal(o.unpack_base3(p, K), o.unpack_ternary(o.pack_ternary(c), K))
    # the all-zero row is the digit-1 byte everywhere, padding included
    assert set(o.pack_base3(np.zeros((1, 8192), np.int8)).ravel().tolist()) == {128}


def test_base3_bytewise_definition():
    # decode one random row digit by digit from the layout definition (plain
    # integer division of v, recovered from the byte by trying every v)
    rng = np.random.default_rng(10)
    K = 128
    c = rng.integers(-1, 2, (1, K)).astype(np.int8)
    p = o.pack_base3(c)[0]
    inv = {-(-256 * v // 243): v for v in range(243)}
    for k in range(K):
        g, r = divmod(k, 20)
        L, b = divmod(r, 4)
        v = inv[int(p[4 * g + b])]
        assert (v // 3 ** (4 - L)) % 3 - 1 == c[0, k]


# ---------------------------------------------------------------------------
# Packed 4-bit activations (P1 Step 4: n // 2 bytes; the nibble order is this
# library's)
# ---------------------------------------------------------------------------

def test_int4_layout_golden():
    g = json.load(open(os.path.join(GOLDEN, "int4_layout.json")))
    q = np.array([g["codes"]], dtype=np.int8)
    p = o.pack_int4(q)
    assert p.tolist() == [g["packed_bytes"]]
    assert np.array_equal(o.unpack_int4(p, q.shape[1]), q)


def test_int4_nibble_by_nibble_and_roundtrip():
    rng = np.random.default_rng(11)
    for M, K in [(1, 64), (3, 4096), (5, 8192)]:
        q = rng.integers(-8, 8, (M, K)).astype(np.int8)
        p = o.pack_int4(q)
        assert p.shape == (M, K // 2) and p.nbytes * 2 == q.size
        assert np.array_equal(o.unpack_int4(p, K), q)
        # nibble by nibble with explicit sign extension
        for m, k in [(0, 0), (0, 1), (M - 1, K - 1), (M - 1, K - 2)]:
            nib = (int(p[m, k // 2]) >> (4 * (k % 2))) & 0xF
            assert (nib - 16 if nib & 8 else nib) == q[m, k]
    with pytest.raises(ValueError):
        o.pack_int4(np.array([[8, 0]], dtype=np.int8))


def test_int4_of_the_a48_quantiser_output():
    # the a4.8 quantiser's codes (Q = 7) fit the nibbles and survive packing
    from bitlinear_bl_forward_b200.inputs import WORKLOADS, layer_inputs
    w = WORKLOADS["a48"]
    X, _ = layer_inputs(w, 0, M=4)
    q, _ = o.act_quant(X, 4)
    assert q.min() >= -8 and q.max() <= 7
    assert np.array_equal(o.unpack_int4(o.pack_int4(q), q.shape[1]), q)


# ---------------------------------------------------------------------------
# [P2] eq. (2), [P1] section 1: activation quantisation
# ---------------------------------------------------------------------------

def test_act_quant_hand_cases():
    x = to_bf16_bits_exact([[1, -2, 0.5, 4],
                            [127, 2.5, 3.5, -0.5],
                            [0, 0, 0, 0],
                            [3, 1.5, -3, 0.75]])
    q, s = o.act_quant(x, 8)
    assert s[0] == np.float32(31.75)
    assert q[0].tolist() == [32, -64, 16, 127]      # -63.5 ties to -64
    assert s[1] == np.float32(1.0)
    assert q[1].tolist() == [127, 2, 4, 0]          # 2.5 -> 2, 3.5 -> 4, -0.5 -> -0
    assert s[2] == np.float32(127) / np.float32(1e-5)
    assert q[2].tolist() == [0, 0, 0, 0]
    # fp32 product decides the code: s = f32(127/3) = 11097429 * 2^-18 and
    # 1.5*s = 16646143.5 * 2^-18 is a tie in fp32 that rounds (to even) up
    # to 63.5, then rint(63.5) = 64.  In exact arithmetic it would be 63.
    assert s[3] == np.float32(11097429 * 2.0 ** -18)
    assert q[3].tolist() == [127, 64, -127, 32]
    assert float(Fraction(3, 2) * Fraction(127, 3)) == 63.5


def test_act_quant_int4_hand_cases():
    x = to_bf16_bits_exact([[7, -3.5, 2.5, 0.375, -7, 0]])
    q, s = o.act_quant(x, 4)
    assert s[0] == np.float32(1.0)
    assert q[0].tolist() == [7, -4, 2, 0, -7, 0]


def test_act_quant_invariants():
    rng = np.random.default_rng(9)
    xf = rng.standard_normal((64, 512)).astype(np.float32)
    xf[:, :3] *= 20
    xf[5] = 0
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)     # truncation is fine: any bf16 data
    for bits in (8, 4):
        Q = o.QMAX[bits]
        q, s = o.act_quant(x, bits)
        assert np.all(np.abs(q.astype(np.int32)) <= Q)          # never -Q-1
        nz = np.any(o.bf16_bits_to_f32(x) != 0, axis=1)
        assert np.all(np.max(np.abs(q[nz].astype(np.int32)), axis=1) == Q)
        assert np.all(q[~nz] == 0)


def test_a4_divide_form_is_close():
    # P1's literal form x / (a/7) and the multiply form x * (7/a) agree on
    # nearly every code; where they differ, by exactly one (a tie moved by
    # one rounding).
    rng = np.random.default_rng(10)
    z = rng.standard_normal((256, 1024)).astype(np.float32)
    x = (np.maximum(z, 0) ** 2).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    q1, _ = o.act_quant(xb, 4)
    q2, _ = o.act_quant(xb, 4, a4_divide_form=True)
    d = np.abs(q1.astype(np.int32) - q2.astype(np.int32))
    assert d.max() <= 1
    assert np.mean(d) < 1e-3


# ---------------------------------------------------------------------------
# [P2] eq. (3), "Why 1.58 Bits?": integer matmul and rescale
# ---------------------------------------------------------------------------

def naive_acc(q, c):
    M, K = q.shape
    N = c.shape[0]
    out = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            t = 0
            for k in range(K):
                t += int(q[m, k]) * int(c[n, k])
            out[m][n] = t
    return np.array(out, dtype=np.int64)


def test_matmul_brute_force_and_add_sub_form():
    rng = np.random.default_rng(11)
    for (M, K, N) in [(1, 16, 1), (3, 64, 5), (7, 48, 9)]:
        q = rng.integers(-128, 128, (M, K)).astype(np.int8)
        c = rng.integers(-1, 2, (N, K)).astype(np.int8)
        acc = o.matmul_i32(q, c)
        assert np.array_equal(acc, naive_acc(q, c))
        # ternary weight adds (+1), subtracts (-1) or skips (0) the activation
        for m in range(M):
            for n in range(N):
                plus = int(q[m][c[n] == 1].astype(np.int64).sum())
                minus = int(q[m][c[n] == -1].astype(np.int64).sum())
                assert acc[m, n] == plus - minus


def test_matmul_extremes():
    K = 8192
    q = np.full((2, K), 127, np.int8)
    q[1] = -127
    c = np.ones((2, K), np.int8)
    c[1] = -1
    acc = o.matmul_i32(q, c)
    assert acc.tolist() == [[127 * K, -127 * K], [-127 * K, 127 * K]]


def test_rescale_against_exact_rational():
    rng = np.random.default_rng(12)
    acc = rng.integers(-300000, 300000, (5, 7)).astype(np.int32)
    s = (np.float32(127) / (np.abs(rng.standard_normal(5)) + 0.1).astype(np.float32)).astype(np.float32)
    g = np.float32(0.0123)
    y64, y32 = o.rescale(acc, g, s)
    for m in range(5):
        for n in range(7):
            exact = Fraction(int(acc[m, n])) * Fraction(float(g)) / Fraction(float(s[m]))
            assert abs(Fraction(float(y64[m, n])) - exact) <= abs(exact) * Fraction(1, 1 << 51)
            assert abs(Fraction(float(y32[m, n])) - exact) <= abs(exact) * Fraction(1, 1 << 22)


def test_dequantized_float_matmul_brute_force():
    # The pages' simulated integer GEMM (F.linear on dequantised operands)
    # equals the integer path: y = (q/s) . (c*gamma)^T, in exact arithmetic.
    rng = np.random.default_rng(13)
    M, K, N = 4, 64, 6
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xf = rng.standard_normal((M, K)).astype(np.float32)
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    r = o.forward(x, W)
    g = Fraction(float(r["gamma"]))
    for m in range(M):
        sm = Fraction(float(r["s"][m]))
        for n in range(N):
            exact = sum(Fraction(int(r["q"][m, k])) / sm * (int(r["codes"][n, k]) * g) for k in range(K))
            assert abs(Fraction(float(r["y64"][m, n])) - exact) <= abs(exact) * Fraction(1, 1 << 50)


def test_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    W = np.array([g["W"]], np.float32)
    x = to_bf16_bits_exact([g["x"]])
    r = o.forward(x, W)
    assert r["gamma"] == np.float32(g["gamma"])
    assert r["codes"][0].tolist() == g["codes"]
    assert r["s"][0] == np.float32(g["s"])
    assert r["q"][0].tolist() == g["q"]
    assert int(r["acc"][0, 0]) == g["acc"]
    exact = Fraction(g["y_exact_num"]) / Fraction(g["y_exact_den"])
    assert abs(Fraction(float(r["y64"][0, 0])) - exact) <= exact * Fraction(1, 1 << 50)
    assert int(r["Y"][0, 0]) == g["Y_bf16_bits"]


def test_zero_row_and_zero_weights():
    W = np.zeros((3, 32), np.float32)
    x = to_bf16_bits_exact([[0.0] * 32, [1.0] * 32])
    r = o.forward(x, W)
    assert r["gamma"] == o.EPS
    assert np.all(r["codes"] == 0)
    assert np.all(r["acc"] == 0)
    assert np.all(r["Y"] == 0)


# ---------------------------------------------------------------------------
# P3 section "2. Squared ReLU Activation": the down projection's input
# ---------------------------------------------------------------------------

def test_relu2_hand_cases():
    # ReLU^2(x) = max(0, x)^2; gated: times the up output
    g = to_bf16_bits_exact([[-3.0, -0.0, 0.5, 3.0, 1.5]])
    u = to_bf16_bits_exact([[7.0, 2.0, -4.0, -1.5, 0.25]])
    h = o.relu2_input(g)
    assert h.dtype == np.float32
    assert h.tolist() == [[0.0, 0.0, 0.25, 9.0, 2.25]]
    hg = o.relu2_input(g, u)
    assert hg.tolist() == [[0.0, 0.0, -1.0, -13.5, 0.5625]]


def test_relu2_is_exact_for_bf16_inputs():
    # bf16 has 8 significant bits: g^2 (16 bits) and g^2 * u (24 bits) are
    # exact in fp32, so h equals the exact rational product
    rng = np.random.default_rng(21)
    vals = rng.standard_normal((4, 64)).astype(np.float32) * 3
    ub = rng.standard_normal((4, 64)).astype(np.float32)
    gb = (vals.view(np.uint32) >> 16).astype(np.uint16)
    uu = (ub.view(np.uint32) >> 16).astype(np.uint16)
    h = o.relu2_input(gb, uu)
    g = gb.astype(np.uint32) << 16
    u = uu.astype(np.uint32) << 16
    for i in range(4):
        for k in range(64):
            gf = Fraction(float(np.uint32(g[i, k]).view(np.float32)))
            uf = Fraction(float(np.uint32(u[i, k]).view(np.float32)))
            exact = (max(gf, Fraction(0)) ** 2) * uf
            assert Fraction(float(h[i, k])) == exact


def test_act_quant_values_hand_case_and_agrees_on_bf16():
    # h = [0.5, -2, 1]: a = 2, s = 63.5, h*s = [31.75, -127, 63.5] -> 32, -127, 64 (tie to even)
    q, s = o.act_quant_values(np.array([[0.5, -2.0, 1.0]], np.float32))
    assert s[0] == np.float32(63.5)
    assert q.tolist() == [[32, -127, 64]]
    # on bf16-representable values it is the (separately pinned) act_quant
    rng = np.random.default_rng(5)
    xb = (rng.standard_normal((6, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    for bits in (8, 4):
        q1, s1 = o.act_quant(xb, bits)
        q2, s2 = o.act_quant_values(o.bf16_bits_to_f32(xb), bits)
        assert np.array_equal(q1, q2) and np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def test_forward_relu2_matches_dequantized_brute_force():
    # y = sum_k c[n,k] * q[m,k] * gamma / s_m, against exact rationals
    rng = np.random.default_rng(8)
    M, K, N = 3, 64, 5
    gb = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    out = o.forward_relu2(gb, None, W)
    h = out["h"]
    assert np.all(h >= 0) and np.any(h == 0)     # ReLU^2 is sparse and non-negative
    for m in range(M):
        a = max(Fraction(float(v)) for v in h[m])
        for n in range(N):
            acc = sum(int(out["codes"][n, k]) * int(out["q"][m, k]) for k in range(K))
            assert acc == out["acc"][m, n]
            exact = Fraction(acc) * Fraction(float(out["gamma"])) / Fraction(float(out["s"][m]))
            assert abs(float(exact) - out["y64"][m, n]) <= 1e-12 * max(1.0, abs(float(exact)))
        # s_m is 127 / max_k h, correctly rounded to fp32
        assert out["s"][m] == o.round_rational_to_f32(127 * a.denominator, a.numerator)


# ---------------------------------------------------------------------------
# variants the pages print: per-tensor activation scale (P3 section 1) and bias
# ---------------------------------------------------------------------------

def test_act_quant_per_tensor_hand_case():
    # rows [1, 2] and [4, -8]: a = 8 over the tensor, s = 127/8 = 15.875 (exact)
    x = to_bf16_bits_exact([[1.0, 2.0], [4.0, -8.0]])
    q, s = o.act_quant_per_tensor(x)
    assert s.tolist() == [15.875, 15.875]
    # 15.875 -> 16, 31.75 -> 32, 63.5 -> 64 (tie to even), -127
    assert q.tolist() == [[16, 32], [64, -127]]


def test_act_quant_per_tensor_reduces_to_per_token():
    rng = np.random.default_rng(12)
    x1 = (rng.standard_normal((1, 256)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    for bits in (8, 4):
        assert np.array_equal(o.act_quant_per_tensor(x1, bits)[0], o.act_quant(x1, bits)[0])
    # rows that share the same absmax: per-tensor equals per-token
    x = rng.standard_normal((5, 128)).astype(np.float32)
    x[:, 7] = 9.0
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    qa, sa = o.act_quant_per_tensor(xb)
    qb, sb = o.act_quant(xb)
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)
    # otherwise every row uses the smallest per-token scale
    xr = (rng.standard_normal((5, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.all(o.act_quant_per_tensor(xr)[1] == o.act_quant(xr)[1].min())


def test_forward_ex_bias_hand_case():
    # the worked example (y32 = 143 * f32(gamma / s)) plus a bias of -0.25
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    W = np.array([ex["W"]], np.float32)
    x = to_bf16_bits_exact([ex["x"]])
    plain = o.forward(x, W)
    out = o.forward_ex(x, W, bias=np.array([-0.25], np.float32))
    assert out["acc"][0, 0] == 143
    assert out["y32"][0, 0] == np.float32(np.float32(plain["y32"][0, 0]) + np.float32(-0.25))
    assert abs(out["y64"][0, 0] - (plain["y64"][0, 0] - 0.25)) < 1e-15


# ---------------------------------------------------------------------------
# P3 section "3. Sub-Layer Normalization (SubLN)": RMSNorm before the absmax
# ---------------------------------------------------------------------------

def _bf16_of(values):
    """Round-to-nearest-even bf16 bit patterns, computed by torch (independent
    of the oracle's own rounding helper)."""
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_exact_square_sum_against_fractions():
    rng = np.random.default_rng(41)
    # every exponent class, subnormals and zeros included
    bits = rng.integers(0, 0x7F80, size=700).astype(np.uint16)
    bits[:40] = rng.integers(0, 0x80, size=40)          # subnormals and zero
    bits[40:60] = 0
    signs = rng.integers(0, 2, size=bits.size).astype(np.uint16) << 15
    bits = bits | signs
    vals = o.bf16_bits_to_f32(bits).astype(np.float64)
    exact = sum((Fraction(float(v)) ** 2 for v in vals), Fraction(0))
    assert Fraction(o.exact_square_sum(bits), 1 << 266) == exact


def test_rms_norm_closed_form_rms_of_one_and_seven():
    # half the entries 1, half -7: mean of squares (1 + 49) / 2 = 25, RMS 5
    K = 64
    x = to_bf16_bits_exact([1.0] * (K // 2) + [-7.0] * (K // 2))[None, :]
    r = o.rms_norm(x, eps=1e-30)
    assert r["ms"][0] == np.float32(25.0) and r["r"][0] == np.float32(5.0)
    want = _bf16_of([1.0 / 5.0] * (K // 2) + [-7.0 / 5.0] * (K // 2))
    assert np.array_equal(r["xn"][0], want)


def test_rms_norm_unit_rows_map_to_themselves():
    rng = np.random.default_rng(5)
    x = to_bf16_bits_exact(rng.choice([-1.0, 1.0], size=(3, 256)))
    r = o.rms_norm(x, eps=1e-30)
    assert np.all(r["ms"] == 1.0) and np.all(r["r"] == 1.0)
    assert np.array_equal(r["xn"], x)


def test_rms_norm_power_of_two_scale_invariance():
    # x -> 2^j x with eps -> 4^j eps scales ms by 4^j and r by 2^j exactly,
    # so the normalised values do not move
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 320)).astype(np.float32)
    xb = _bf16_of(x)
    base = o.rms_norm(xb, eps=2.0 ** -20)
    for j in (-9, -1, 3, 12):
        xs = _bf16_of(o.bf16_bits_to_f32(xb) * np.float32(2.0 ** j))
        r = o.rms_norm(xs, eps=2.0 ** (-20 + 2 * j))
        assert np.array_equal(r["ms"], (base["ms"] * np.float32(4.0 ** j)).astype(np.float32))
        assert np.array_equal(r["r"], (base["r"] * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(r["xn"], base["xn"])


def test_rms_norm_mean_of_squares_is_rounded_once_from_the_exact_sum():
    # K = 128: 64 ones and one 2^-9 give sum 64 + 2^-18, mean 0.5 + 2^-25,
    # exactly halfway between the fp32 neighbours 0.5 and 0.5 + 2^-24: ties
    # to even -> 0.5.  One more entry 2^-60 puts the exact mean just above the
    # midpoint -> 0.5 + 2^-24, which a float64 sum would miss.
    K = 128
    v = np.zeros(K, np.float32)
    v[:64] = 1.0
    v[64] = 2.0 ** -9
    r = o.rms_norm(to_bf16_bits_exact(v)[None, :], eps=2.0 ** -40)
    assert r["ms"][0] == np.float32(0.5)
    v[65] = 2.0 ** -60
    r = o.rms_norm(to_bf16_bits_exact(v)[None, :], eps=2.0 ** -40)
    assert r["ms"][0] == np.float32(0.5 + 2.0 ** -24)
    assert np.float32(np.sum(v.astype(np.float64) ** 2) / K) == np.float32(0.5)


def test_rms_norm_weight():
    rng = np.random.default_rng(7)
    xb = _bf16_of(rng.standard_normal((2, 128)))
    plain = o.rms_norm(xb, eps=1e-6)
    two = o.rms_norm(xb, to_bf16_bits_exact(np.full(128, 2.0)), eps=1e-6)
    assert np.array_equal(o.bf16_bits_to_f32(two["xn"]), 2.0 * o.bf16_bits_to_f32(plain["xn"]))
    w = np.ones(128, np.float32)
    w[::3] = 0.0
    z = o.rms_norm(xb, to_bf16_bits_exact(w), eps=1e-6)
    assert np.all(o.bf16_bits_to_f32(z["xn"])[:, ::3] == 0.0)
    assert np.array_equal(z["xn"][:, 1::3], plain["xn"][:, 1::3])


def test_rms_norm_against_float64_brute_force():
    rng = np.random.default_rng(8)
    M, K = 6, 448
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-8, 8, size=(M, 1)))).astype(np.float32)
    x[:, rng.integers(0, K, 4)] *= 30.0
    xb = _bf16_of(x)
    wb = _bf16_of(rng.uniform(0.5, 1.5, size=K))
    eps = 1e-5
    r = o.rms_norm(xb, wb, eps=eps)
    x64 = o.bf16_bits_to_f32(xb).astype(np.float64)
    w64 = o.bf16_bits_to_f32(wb).astype(np.float64)
    ref = x64 / np.sqrt(np.mean(x64 ** 2, axis=1, keepdims=True) + eps) * w64
    got = o.bf16_bits_to_f32(r["xn"]).astype(np.float64)
    ulp = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)   # one bf16 ulp at |ref|
    assert np.all(np.abs(got - ref) <= ulp)


def test_rms_norm_zero_row_and_bad_eps():
    x = np.zeros((2, 64), np.uint16)
    x[1, 5] = 0x3F80
    r = o.rms_norm(x, eps=0.25)
    assert r["ms"][0] == 0.0 and r["r"][0] == np.float32(0.5)
    assert np.all(r["xn"][0] == 0)
    # one entry 1 of 64: ms = 1/64, r = sqrt(1/64 + 0.25)
    assert r["ms"][1] == np.float32(1.0 / 64.0)
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(ValueError):
            o.rms_norm(x, eps=bad)


def test_forward_rmsnorm_is_forward_on_the_normalised_input():
    rng = np.random.default_rng(9)
    xb = _bf16_of(rng.standard_normal((3, 128)) * 4.0)
    W = rng.standard_normal((32, 128)).astype(np.float32)
    got = o.forward_rmsnorm(xb, W, eps=1e-5, bits=4)
    ref = o.forward(o.rms_norm(xb, eps=1e-5)["xn"], W, bits=4)
    assert np.array_equal(got["Y"], ref["Y"]) and np.array_equal(got["q"], ref["q"])


def test_round_rational_overflow_boundary():
    # IEEE round to nearest: the largest fp32 is (2^24 - 1) 2^104; values
    # from the midpoint (2^128 - 2^103) up round to infinity, below it to the
    # largest fp32
    fmax = np.finfo(np.float32).max
    assert o.round_rational_to_f32((1 << 128) - (1 << 104), 1) == fmax
    assert o.round_rational_to_f32((1 << 128) - (1 << 103) - 1, 1) == fmax
    assert np.isinf(o.round_rational_to_f32((1 << 128) - (1 << 103), 1))
    assert np.isinf(o.round_rational_to_f32(1 << 128, 1))
    assert np.isinf(o.round_rational_to_f32(3 << 300, 7))


# ---------------------------------------------------------------------------
# LayerNorm (non-affine) ahead of the quantiser: "BitNet b1.58: The 1-Bit
# Ternary LLM Architecture Guide", BitLinear code listing, forward step 1
# ---------------------------------------------------------------------------

def _f32_round_signed(fr: Fraction) -> np.float32:
    """fp32 round-to-nearest-even of a rational (symmetric in the sign)."""
    v = o.round_rational_to_f32(abs(fr.numerator), fr.denominator)
    return np.float32(-v) if fr < 0 else v


def test_layer_norm_hand_worked_golden():
    with open(os.path.join(os.path.dirname(__file__), "golden", "layernorm_example.json")) as f:
        g = json.load(f)
    xb = to_bf16_bits_exact(np.asarray(g["x"], np.float32))
    r = o.layer_norm(xb, eps=g["eps"])
    assert np.array_equal(r["mean"], np.asarray(g["mean"], np.float32))
    assert np.array_equal(r["var"], np.asarray(g["var"], np.float32))
    assert np.array_equal(r["xn"], np.asarray(g["xn_bf16_bits"], np.uint16))


def test_exact_sum_against_fractions():
    rng = np.random.default_rng(42)
    bits = rng.integers(0, 0x7F80, size=900).astype(np.uint16)
    bits[:50] = rng.integers(0, 0x80, size=50)          # subnormals and zero
    bits[50:70] = 0
    bits |= rng.integers(0, 2, size=bits.size).astype(np.uint16) << 15
    vals = o.bf16_bits_to_f32(bits).astype(np.float64)
    exact = sum((Fraction(float(v)) for v in vals), Fraction(0))
    assert Fraction(o.exact_sum(bits), 1 << 133) == exact
    # cancellation to exactly zero across the whole exponent range
    both = np.concatenate([bits, bits ^ np.uint16(0x8000)])
    assert o.exact_sum(both) == 0


def test_layer_norm_against_two_pass_fractions():
    # textbook two-pass definition in exact rationals: mu = sum/K, var =
    # sum (x - mu)^2 / K; then every fp32 step rounded from its exact value
    rng = np.random.default_rng(43)
    for K in (2, 3, 5, 16, 64):
        x = (rng.standard_normal((3, K)) * np.exp(rng.uniform(-6, 6, size=(3, 1))) + rng.uniform(-4, 4, (3, 1)))
        xb = _bf16_of(x)
        eps = 1e-5
        r = o.layer_norm(xb, eps=eps)
        xs = o.bf16_bits_to_f32(xb)
        for m in range(3):
            fr = [Fraction(float(v)) for v in xs[m]]
            mu = sum(fr, Fraction(0)) / K
            var = sum(((v - mu) ** 2 for v in fr), Fraction(0)) / K
            assert r["mean"][m] == _f32_round_signed(mu)
            assert r["var"][m] == o.round_rational_to_f32(var.numerator, var.denominator)
            v32 = _f32_round_signed(Fraction(float(r["var"][m])) + Fraction(float(np.float32(eps))))
            r32 = np.float32(math.sqrt(float(v32)))   # IEEE sqrt of a double holding an fp32, then rounded
            assert r["r"][m] == r32
            for k in range(K):
                d = _f32_round_signed(fr[k] - Fraction(float(r["mean"][m])))
                t = _f32_round_signed(Fraction(float(d)) / Fraction(float(r32)))
                assert r["t"][m, k] == t


def test_layer_norm_mean_rounds_once_ties_to_even():
    # K = 64: 64 and 2^-18 sum to 64 + 2^-18, mean 1 + 2^-24, halfway between
    # 1 and 1 + 2^-23: ties to even -> 1.  64 + 2^-17 + 2^-18 gives mean
    # 1 + 3 2^-24, halfway between 1 + 2^-23 and 1 + 2^-22: even -> 1 + 2^-22.
    # One more entry 2^-100 lifts the first case just above its midpoint
    # (-> 1 + 2^-23), which a float64 sum would not see.
    v = np.zeros(64, np.float32)
    v[0], v[1] = 64.0, 2.0 ** -18
    assert o.layer_norm(to_bf16_bits_exact(v)[None, :])["mean"][0] == np.float32(1.0)
    v[2] = 2.0 ** -100
    assert o.layer_norm(to_bf16_bits_exact(v)[None, :])["mean"][0] == np.float32(1.0 + 2.0 ** -23)
    assert np.float32(np.sum(v.astype(np.float64)) / 64) == np.float32(1.0)
    v[1], v[2] = 2.0 ** -17, 2.0 ** -18
    assert o.layer_norm(to_bf16_bits_exact(v)[None, :])["mean"][0] == np.float32(1.0 + 2.0 ** -22)
    # negative mirror image
    assert o.layer_norm(to_bf16_bits_exact(-v)[None, :])["mean"][0] == np.float32(-1.0 - 2.0 ** -22)


def test_layer_norm_constant_and_zero_rows():
    x = to_bf16_bits_exact(np.array([[3.5] * 128, [0.0] * 128, [-2.0 ** 100] * 128], np.float32))
    r = o.layer_norm(x, eps=0.25)
    assert np.array_equal(r["var"], np.zeros(3, np.float32))
    assert r["mean"][0] == np.float32(3.5) and r["mean"][1] == 0.0
    assert r["mean"][2] == o.bf16_bits_to_f32(x[2:3, 0])[0]
    assert np.all(r["r"] == np.float32(0.5)) and np.all(r["xn"] == 0)
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(ValueError):
            o.layer_norm(x, eps=bad)


def test_layer_norm_power_of_two_scale_and_integer_shift():
    rng = np.random.default_rng(44)
    xb = _bf16_of(rng.standard_normal((4, 320)))
    base = o.layer_norm(xb, eps=2.0 ** -20)
    for j in (-9, -1, 3, 12):
        xs = _bf16_of(o.bf16_bits_to_f32(xb) * np.float32(2.0 ** j))
        r = o.layer_norm(xs, eps=2.0 ** (-20 + 2 * j))
        assert np.array_equal(r["mean"], (base["mean"] * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(r["var"], (base["var"] * np.float32(4.0 ** j)).astype(np.float32))
        assert np.array_equal(r["xn"], base["xn"])
    # integers in [-100, 100] shifted by 64 stay exact in bf16: the exact
    # variance does not move
    xi = rng.integers(-100, 101, size=(3, 192)).astype(np.float32)
    a, b = o.layer_norm(to_bf16_bits_exact(xi)), o.layer_norm(to_bf16_bits_exact(xi + 64.0))
    assert np.array_equal(a["var"], b["var"])


def test_layer_norm_against_torch_float64():
    # the library's layer_norm in float64 on the same bf16 inputs (biased
    # variance, eps inside the square root); the oracle's fp32 steps stay
    # within a few fp32 roundings of it
    rng = np.random.default_rng(45)
    M, K = 6, 448
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-8, 8, size=(M, 1)))
         + rng.uniform(-3, 3, size=(M, 1)) * np.exp(rng.uniform(-8, 8, size=(M, 1))))
    x[:, rng.integers(0, K, 4)] *= 30.0
    xb = _bf16_of(x)
    eps = 1e-5
    r = o.layer_norm(xb, eps=eps)
    x64 = torch.from_numpy(o.bf16_bits_to_f32(xb).astype(np.float64))
    ref = torch.nn.functional.layer_norm(x64, (K,), eps=float(np.float32(eps))).numpy()
    mu = np.abs(r["mean"].astype(np.float64))[:, None]
    rr = r["r"].astype(np.float64)[:, None]
    tol = 4 * 2.0 ** -24 * ((np.abs(x64.numpy()) + mu) / rr + np.abs(ref))
    assert np.all(np.abs(r["t"].astype(np.float64) - ref) <= tol)
    # the unbiased (1/(K-1)) variance is measurably different
    unb = (x64.numpy() - x64.numpy().mean(1, keepdims=True)) / np.sqrt(x64.numpy().var(1, ddof=1, keepdims=True) + eps)
    assert np.any(np.abs(r["t"].astype(np.float64) - unb) > tol)


def test_forward_layernorm_is_forward_on_the_normalised_input():
    rng = np.random.default_rng(46)
    xb = _bf16_of(rng.standard_normal((3, 128)) * 4.0 + 2.0)
    W = rng.standard_normal((32, 128)).astype(np.float32)
    got = o.forward_layernorm(xb, W, eps=1e-5, bits=4)
    ref = o.forward(o.layer_norm(xb, eps=1e-5)["xn"], W, bits=4)
    assert np.array_equal(got["Y"], ref["Y"]) and np.array_equal(got["q"], ref["q"])
