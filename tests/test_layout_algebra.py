"""CPU check of the integer identity the one-token kernels rely on.

The 2-bit rows store u = code + 1 at bits [8b + 2j, 8b + 2j + 2) of 32-bit
word g (weight k = 16g + 4j + b).  The kernels take, per word, the four
masked slices w & (0x03030303 << 2j) -- each byte holds u * 4^j -- into four
unsigned-by-signed four-way dot products with the matching token codes,
fold the four sums as acc0 + acc1/4 + acc2/16 + acc3/64 and start from minus
the sum of the codes they cover (per lane in the column-split modes, per
256-code block in the row-lane mode).  This restates that arithmetic in
plain integers on the oracle's packed bytes and checks it against the
oracle's exact matmul (the BitLinear matmul of "BitNet b1.58: The 1-Bit
Ternary LLM Architecture Guide", eq. (3)), for both block splits, so the
decomposition is exact independently of any GPU.
"""

import numpy as np
import pytest

from oracle import bitlinear_oracle as o


def dp4a_us(a_words, b_words):
    """Sum over the four bytes of unsigned a times signed b (per word, int64)."""
    a = a_words.astype(np.uint32)
    b = b_words.astype(np.uint32)
    s = np.zeros(a.shape, dtype=np.int64)
    for byte in range(4):
        ab = ((a >> np.uint32(8 * byte)) & np.uint32(0xFF)).astype(np.int64)
        bb = ((b >> np.uint32(8 * byte)) & np.uint32(0xFF)).astype(np.int64)
        bb = np.where(bb >= 128, bb - 256, bb)
        s += ab * bb
    return s


def slice_fold_dot(words, q_row, block_words):
    """words: uint32 [N, W] (a packed row each); q_row: int8 [16 W].
    Sum over blocks of block_words words: -sum(q of the block) + folded slices."""
    N, W = words.shape
    qb = q_row.astype(np.int8).view(np.uint8).reshape(W, 4, 4)   # [g, j, b]
    act = np.zeros((W, 4), dtype=np.uint32)                      # slice j of word g: 4 codes
    for j in range(4):
        for b in range(4):
            act[:, j] |= qb[:, j, b].astype(np.uint32) << np.uint32(8 * b)
    total = np.zeros(N, dtype=np.int64)
    for w0 in range(0, W, block_words):
        w1 = min(W, w0 + block_words)
        neg = -int(q_row[16 * w0:16 * w1].astype(np.int64).sum())
        acc = [np.zeros(N, dtype=np.int64) for _ in range(4)]
        acc[0] += neg
        for g in range(w0, w1):
            for j in range(4):
                m = np.uint32(0x03030303 << (2 * j))
                acc[j] += dp4a_us(words[:, g] & m, np.full(N, act[g, j], dtype=np.uint32))
        for j in (1, 2, 3):
            assert np.all(acc[j] % (4 ** j) == 0)      # each slice sum is an exact multiple
        total += acc[0] + acc[1] // 4 + acc[2] // 16 + acc[3] // 64
    return total


@pytest.mark.parametrize("K", [64, 256, 2560, 6912])
@pytest.mark.parametrize("block_words", [16, 32, 8192])   # 256-code blocks, 512-code blocks, whole rows
def test_slice_fold_equals_exact_matmul(K, block_words):
    rng = np.random.default_rng(K + block_words)
    N = 23
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    q = rng.integers(-128, 128, size=(1, K)).astype(np.int8)
    packed = o.pack_ternary(codes)
    words = np.ascontiguousarray(packed).view("<u4")
    got = slice_fold_dot(words, q[0], block_words)
    want = o.matmul_i32(q, codes)[0].astype(np.int64)
    assert np.array_equal(got, want)


def test_extreme_codes_stay_exact():
    # every weight +1 or -1 and every code at -128 / 127: the largest sums
    K = 2560
    for c, qv in ((1, 127), (-1, 127), (1, -128), (-1, -128)):
        codes = np.full((2, K), c, dtype=np.int8)
        q = np.full((1, K), qv, dtype=np.int8)
        words = np.ascontiguousarray(o.pack_ternary(codes)).view("<u4")
        assert np.array_equal(slice_fold_dot(words, q[0], 16), np.full(2, c * qv * K, dtype=np.int64))
