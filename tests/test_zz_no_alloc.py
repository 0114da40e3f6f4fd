"""The allocation-free forward (bl_forward_noalloc).

Some callers cannot allocate device memory or hand the library a workspace,
for example an engine that budgets all device memory once at start-up and
gives an operator only its input and output buffers.  bl_forward_noalloc
serves them: it keeps the tensor-core path's scratch in one static device array
of the library.  These tests call it through the C ABI and compare it with
bl_forward, which takes a caller workspace.  Both run the same kernels on the
same inputs, so the outputs must be bit-identical.  The shapes reach the decode
path (one token), both activation quantisers (many short rows; few long rows),
both tensor-core GEMMs, and a shape whose int8 codes fill the scratch exactly.
Consecutive calls with different shapes check that a call does not depend on
what the previous call left in the shared array.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from bitlinear_bl_forward_b200 import bl
from bitlinear_bl_forward_b200 import build as blbuild
from bitlinear_bl_forward_b200.inputs import random_case
from tests.gpu_helpers import x_to_dev

SCRATCH_LIMIT = 8


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L = bl.lib()
    bl.bl_device_status(clear=True)
    cases = [
        (300, 2560, 700, 8, 21),      # warp-per-row quantiser, CTA-pair GEMM
        (64, 512, 384, 4, 22),        # one-SM GEMM, 4-bit codes
        (1, 2560, 6912, 8, 23),       # decode path (no scratch used)
        (3, 8192, 256, 8, 24),        # few long rows: CTA-per-row quantiser
        (2048, 8192, 320, 8, 25),     # M * K = 16 MiB: the scratch limit exactly
    ]
    for M, K, N, bits, seed in cases:
        X, W = random_case(M, K, N, seed)
        Wp, gamma = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        Xd = x_to_dev(X)
        ref = bl.bl_forward(Xd, Wp, gamma, N, bits)
        for _ in range(2):
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            st = L.bl_forward_noalloc(Xd.data_ptr(), M, K, N, Wp.data_ptr(), gamma.data_ptr(), bits, Y.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
            assert st == 0, bl.STATUS_NAMES.get(st, st)
            torch.cuda.synchronize()
            assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), f"M={M} K={K} N={N}"
    assert bl.bl_device_status(clear=True) == (0, 0)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # rejected on the host before any launch (the pointers are never used)
    blbuild.build()
    L = bl.lib()
    A = 0x10000
    assert L.bl_forward_noalloc(A, 4096, 8192, 8, A, A, 8, A, None) == SCRATCH_LIMIT   # M*K = 32 MiB
    assert L.bl_forward_noalloc(A, 8193, 64, 8, A, A, 8, A, None) == SCRATCH_LIMIT     # M > 8192
    assert L.bl_status_string(SCRATCH_LIMIT).startswith(b"shape exceeds")
