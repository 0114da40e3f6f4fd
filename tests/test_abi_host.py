"""Host-side checks of the C ABI that need no GPU.

* the library loads and exports every entry point include/bitlinear.h declares;
* the Python binding mirrors exactly those names;
* argument validation rejects bad calls before any CUDA call.

Every validation call below carries at least one invalid argument, so nothing
is ever launched (the pointers are fake and are never dereferenced).
"""

import ctypes
import os
import re

import pytest

from bitlinear_bl_forward_b200 import bl
from bitlinear_bl_forward_b200 import build as blbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")

OK, INVALID, SHAPE, ALIGN, UNSUP, CUDA, TIMEOUT, WS = range(8)
A = 0x10000      # fake, 16-byte aligned
U = 0x10001      # fake, misaligned


@pytest.fixture(scope="module")
def L():
    blbuild.build()
    return bl.lib()


def header_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^BL_API\s+[\w\s\*]+?\b(bl_\w+)\s*\(", txt, flags=re.M)))


def test_header_symbols_exported(L):
    syms = header_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(L, s), s
    # and nothing else with the bl_ prefix is bound by Python
    assert sorted(bl.SIGNATURES) == syms


def test_binding_names_match_header():
    for s in header_symbols():
        if s in ("bl_status_string", "bl_version", "bl_quantize_weights_workspace_bytes",
                 "bl_matmul_i32_workspace_bytes"):
            continue
        assert hasattr(bl, s), s


def test_status_strings(L):
    for code in range(8):
        assert L.bl_status_string(code)
    assert L.bl_status_string(99) == b"unknown status"
    assert L.bl_version() >= 100


def test_sizes(L):
    assert L.bl_packed_weight_bytes(6912, 2560) == 6912 * 2560 // 4
    assert L.bl_packed_weight_bytes(28672, 8192) == 58720256
    assert L.bl_forward_workspace_bytes(1, 2560, 6912, 8) == 0
    assert L.bl_forward_workspace_bytes(2, 2560, 6912, 8) == 0
    ws = L.bl_forward_workspace_bytes(4096, 2560, 6912, 8)
    assert ws >= 4096 * 2560 + 2 * 4 * 4096
    assert L.bl_forward_workspace_bytes(4096, 2500, 6912, 8) == 0     # bad shape
    assert L.bl_quantize_weights_workspace_bytes(512, 256) > 0
    assert L.bl_matmul_i32_workspace_bytes(17, 256, 512) >= 17 * 4


@pytest.mark.parametrize("args,want", [
    # (X, M, K, N, Wp, gamma, bits, Y, ws, ws_bytes)
    ((A, 4, 100, 8, A, A, 8, A, A, 1 << 20), SHAPE),       # K % 64
    ((A, 4, 0, 8, A, A, 8, A, A, 1 << 20), SHAPE),
    ((A, 4, 131072, 8, A, A, 8, A, A, 1 << 30), SHAPE),    # K too large
    ((A, 4, 64, 0, A, A, 8, A, A, 1 << 20), SHAPE),        # N <= 0
    ((A, -1, 64, 8, A, A, 8, A, A, 1 << 20), SHAPE),       # M < 0
    ((A, 4, 64, 8, A, A, 2, A, A, 1 << 20), UNSUP),        # bits
    ((A, 4, 64, 8, A, A, 16, A, A, 1 << 20), UNSUP),
    ((None, 4, 64, 8, A, A, 8, A, A, 1 << 20), INVALID),
    ((A, 4, 64, 8, None, A, 8, A, A, 1 << 20), INVALID),
    ((A, 4, 64, 8, A, None, 8, A, A, 1 << 20), INVALID),
    ((A, 4, 64, 8, A, A, 8, None, A, 1 << 20), INVALID),
    ((U, 4, 64, 8, A, A, 8, A, A, 1 << 20), ALIGN),
    ((A, 4, 64, 8, U, A, 8, A, A, 1 << 20), ALIGN),
    ((A, 4, 64, 8, A, A, 8, A, None, 0), WS),              # workspace needed (M > 2)
    ((A, 4, 64, 8, A, A, 8, A, A, 16), WS),                # too small
    ((A, 4, 64, 8, A, A, 8, A, U, 1 << 20), ALIGN),
    ((A, 0, 64, 8, None, None, 8, None, None, 0), OK),     # M == 0: nothing to do
])
def test_forward_validation(L, args, want):
    X, M, K, N, Wp, g, bits, Y, ws, wsb = args
    assert L.bl_forward(X, M, K, N, Wp, g, bits, Y, ws, wsb, None) == want
    assert L.bl_forward_f32(X, M, K, N, Wp, g, bits, Y, ws, wsb, None) == want


def test_quantize_weights_validation(L):
    need = L.bl_quantize_weights_workspace_bytes(8, 64)
    assert L.bl_quantize_weights(A, 8, 60, A, A, A, 1 << 20, None) == SHAPE
    assert L.bl_quantize_weights(A, 0, 64, A, A, A, 1 << 20, None) == SHAPE
    assert L.bl_quantize_weights(A, 1 << 30, 1 << 14, A, A, A, 1 << 20, None) == SHAPE   # N*K >= 2^40... 2^44
    assert L.bl_quantize_weights(None, 8, 64, A, A, A, need, None) == INVALID
    assert L.bl_quantize_weights(A, 8, 64, None, A, A, need, None) == INVALID
    assert L.bl_quantize_weights(A, 8, 64, A, None, A, need, None) == INVALID
    assert L.bl_quantize_weights(U, 8, 64, A, A, A, need, None) == ALIGN
    assert L.bl_quantize_weights(A, 8, 64, A, A, None, need, None) == WS
    assert L.bl_quantize_weights(A, 8, 64, A, A, A, need - 1, None) == WS


def test_other_validation(L):
    assert L.bl_quant_act(A, 4, 64, 3, A, A, None) == UNSUP
    assert L.bl_quant_act(A, 4, 65, 8, A, A, None) == SHAPE
    assert L.bl_quant_act(None, 4, 64, 8, A, A, None) == INVALID
    assert L.bl_quant_act(A, 4, 64, 8, U, A, None) == ALIGN
    assert L.bl_quant_act(None, 0, 64, 8, None, None, None) == OK
    assert L.bl_unpack_weights(A, 8, 48, A, None) == SHAPE
    assert L.bl_unpack_weights(None, 8, 64, A, None) == INVALID
    assert L.bl_unpack_weights(A, 8, 64, U, None) == ALIGN
    assert L.bl_matmul_i32(A, 4, 64, 8, A, A, None, 0, None) == WS
    assert L.bl_matmul_i32(None, 4, 64, 8, A, A, A, 1 << 20, None) == INVALID
    assert L.bl_matmul_i32(A, 4, 64, -8, A, A, A, 1 << 20, None) == SHAPE
    assert L.bl_selftest_wait_timeout(1000, None, None) == INVALID


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    # the binding has no fallback: a missing library is an error
    monkeypatch.setattr(bl, "_lib", None)
    monkeypatch.setattr(bl, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        bl.lib()


def test_grouped_validation(L):
    arr = (bl.BLLinear * 9)()
    for i in range(9):
        arr[i] = bl.BLLinear(A, 1, 64, 8, A, A, A)
    assert L.bl_forward_grouped(9, arr, 8, None, 0, None) == UNSUP          # more than 8 problems
    assert L.bl_forward_grouped(2, None, 8, None, 0, None) == INVALID
    assert L.bl_forward_grouped(2, arr, 3, None, 0, None) == UNSUP
    arr[1] = bl.BLLinear(A, 1, 60, 8, A, A, A)                              # K % 64
    assert L.bl_forward_grouped(2, arr, 8, None, 0, None) == SHAPE
    arr[1] = bl.BLLinear(A, 1, 64, 8, None, A, A)
    assert L.bl_forward_grouped(2, arr, 8, None, 0, None) == INVALID
    arr[1] = bl.BLLinear(U, 1, 64, 8, A, A, A)
    assert L.bl_forward_grouped(2, arr, 8, None, 0, None) == ALIGN
    arr[1] = bl.BLLinear(A, 4, 64, 8, A, A, A)                              # M > 2 needs a workspace
    assert L.bl_forward_grouped(2, arr, 8, None, 0, None) == WS
    assert L.bl_forward_grouped_workspace_bytes(2, arr, 8) >= 4 * 64
    assert L.bl_forward_grouped(0, arr, 8, None, 0, None) == OK


def test_relu2_validation(L):
    need = L.bl_forward_relu2_workspace_bytes(4, 64, 8, 8)
    assert need >= 4 * 64
    assert L.bl_forward_relu2_workspace_bytes(1, 2560, 6912, 8) == 0        # fused into the decode kernel
    assert L.bl_forward_relu2_workspace_bytes(2, 2560, 6912, 8) > 0         # via the tensor-core path
    assert L.bl_forward_relu2_workspace_bytes(1, 16384, 64, 8) > 0          # K beyond the decode kernels
    args = (A, None, 4, 64, 8, A, A, 8, A, A, 1 << 20, None)
    assert L.bl_forward_relu2(A, None, 4, 60, 8, A, A, 8, A, A, 1 << 20, None) == SHAPE
    assert L.bl_forward_relu2(None, None, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == INVALID
    assert L.bl_forward_relu2(A, U, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == ALIGN     # misaligned U
    assert L.bl_forward_relu2(A, None, 4, 64, 8, A, A, 3, A, A, 1 << 20, None) == UNSUP
    assert L.bl_forward_relu2(A, None, 4, 64, 8, A, A, 8, A, None, 0, None) == WS
    assert L.bl_forward_relu2(None, None, 0, 64, 8, None, None, 8, None, None, 0, None) == OK
    assert L.bl_quant_act_relu2(A, None, 4, 65, 8, A, A, None) == SHAPE
    assert L.bl_quant_act_relu2(A, A, 4, 64, 2, A, A, None) == UNSUP
    assert L.bl_quant_act_relu2(A, U, 4, 64, 8, A, A, None) == ALIGN
    assert len(args) == 12


def test_forward_ex_validation(L):
    assert L.bl_forward_ex_workspace_bytes(1, 2560, 6912, 8, 1) == 0
    assert L.bl_forward_ex_workspace_bytes(2, 2560, 6912, 8, 0) >= 2 * 2560
    assert L.bl_forward_ex(A, 4, 64, 8, A, A, 8, 2, None, A, A, 1 << 20, None) == UNSUP      # unknown flag
    assert L.bl_forward_ex(A, 4, 64, 8, A, A, 8, 1, A + 2, A, A, 1 << 20, None) == ALIGN    # bias not 4-byte aligned
    assert L.bl_forward_ex(A, 4, 64, 8, A, A, 8, 1, None, A, None, 0, None) == WS
    assert L.bl_forward_ex(None, 4, 64, 8, A, A, 8, 0, None, A, A, 1 << 20, None) == INVALID
    assert L.bl_forward_ex(A, 4, 100, 8, A, A, 8, 0, None, A, A, 1 << 20, None) == SHAPE
    assert L.bl_forward_ex(None, 0, 64, 8, None, None, 8, 1, None, None, None, 0, None) == OK


def test_rmsnorm_validation(L):
    # the workspace is required for every M (the fused one-token path leaves it unused)
    assert L.bl_forward_rmsnorm_workspace_bytes(1, 2560, 6912, 8) >= 2560
    assert L.bl_forward_rmsnorm_workspace_bytes(4, 64, 8, 8) >= 4 * 64
    assert L.bl_forward_rmsnorm_workspace_bytes(4, 60, 8, 8) == 0
    ok = (A, None, 1e-5, 4, 64, 8, A, A, 8, A, A, 1 << 20, None)
    assert len(ok) == 13
    assert L.bl_forward_rmsnorm(A, None, 1e-5, 4, 60, 8, A, A, 8, A, A, 1 << 20, None) == SHAPE
    assert L.bl_forward_rmsnorm(None, None, 1e-5, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == INVALID
    assert L.bl_forward_rmsnorm(A, U, 1e-5, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == ALIGN   # misaligned weight
    assert L.bl_forward_rmsnorm(A, None, 1e-5, 4, 64, 8, A, A, 5, A, A, 1 << 20, None) == UNSUP
    assert L.bl_forward_rmsnorm(A, None, 1e-5, 1, 64, 8, A, A, 8, A, None, 0, None) == WS
    for bad in (0.0, -1e-5, float("inf"), float("nan")):
        assert L.bl_forward_rmsnorm(A, None, bad, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == INVALID
        assert L.bl_quant_act_rmsnorm(A, None, bad, 4, 64, 8, A, A, None, None) == INVALID
    assert L.bl_forward_rmsnorm(None, None, 1e-5, 0, 64, 8, None, None, 8, None, None, 0, None) == OK
    assert L.bl_quant_act_rmsnorm(A, None, 1e-5, 4, 65, 8, A, A, None, None) == SHAPE
    assert L.bl_quant_act_rmsnorm(A, None, 1e-5, 4, 64, 2, A, A, None, None) == UNSUP
    assert L.bl_quant_act_rmsnorm(A, U, 1e-5, 4, 64, 8, A, A, None, None) == ALIGN
    assert L.bl_quant_act_rmsnorm(A, None, 1e-5, 4, 64, 8, A, A, A + 2, None) == ALIGN       # mean_sq misaligned
    assert L.bl_quant_act_rmsnorm(None, None, 1e-5, 4, 64, 8, A, A, None, None) == INVALID


def test_layernorm_validation(L):
    assert L.bl_forward_layernorm_workspace_bytes(1, 2560, 6912, 8) == L.bl_forward_rmsnorm_workspace_bytes(1, 2560, 6912, 8)
    assert L.bl_forward_layernorm_workspace_bytes(4, 60, 8, 8) == 0
    assert L.bl_forward_layernorm(A, 1e-5, 4, 60, 8, A, A, 8, A, A, 1 << 20, None) == SHAPE
    assert L.bl_forward_layernorm(None, 1e-5, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == INVALID
    assert L.bl_forward_layernorm(U, 1e-5, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == ALIGN
    assert L.bl_forward_layernorm(A, 1e-5, 4, 64, 8, A, A, 5, A, A, 1 << 20, None) == UNSUP
    assert L.bl_forward_layernorm(A, 1e-5, 1, 64, 8, A, A, 8, A, None, 0, None) == WS
    for bad in (0.0, -1e-5, float("inf"), float("nan")):
        assert L.bl_forward_layernorm(A, bad, 4, 64, 8, A, A, 8, A, A, 1 << 20, None) == INVALID
        assert L.bl_quant_act_layernorm(A, bad, 4, 64, 8, A, A, None, None, None) == INVALID
    assert L.bl_forward_layernorm(None, 1e-5, 0, 64, 8, None, None, 8, None, None, 0, None) == OK
    assert L.bl_quant_act_layernorm(A, 1e-5, 4, 65, 8, A, A, None, None, None) == SHAPE
    assert L.bl_quant_act_layernorm(A, 1e-5, 4, 64, 2, A, A, None, None, None) == UNSUP
    assert L.bl_quant_act_layernorm(A, 1e-5, 4, 64, 8, A, A, A + 2, None, None) == ALIGN    # mean misaligned
    assert L.bl_quant_act_layernorm(A, 1e-5, 4, 64, 8, A, A, None, A + 1, None) == ALIGN    # var misaligned
    assert L.bl_quant_act_layernorm(None, 1e-5, 4, 64, 8, A, A, None, None, None) == INVALID


def test_norm_grouped_validation(L):
    import ctypes
    from bitlinear_bl_forward_b200.bl import BLLinear
    arr = (BLLinear * 9)()
    for i in range(9):
        arr[i] = BLLinear(A, 1, 256, 64, A, A, A)
    ws = L.bl_forward_norm_grouped_workspace_bytes(3, arr, 8)
    assert ws >= 256
    assert L.bl_forward_norm_grouped_workspace_bytes(9, arr, 8) == 0
    assert L.bl_forward_norm_grouped(9, arr, 0, None, 1e-5, 8, A, 1 << 20, None) == UNSUP     # > 8 problems
    assert L.bl_forward_norm_grouped(3, arr, 2, None, 1e-5, 8, A, 1 << 20, None) == UNSUP     # unknown norm
    w = (ctypes.c_void_p * 3)(A, A, A)
    assert L.bl_forward_norm_grouped(3, arr, 1, w, 1e-5, 8, A, 1 << 20, None) == INVALID      # LayerNorm has no weight
    assert L.bl_forward_norm_grouped(3, arr, 0, None, 0.0, 8, A, 1 << 20, None) == INVALID    # eps
    assert L.bl_forward_norm_grouped(3, arr, 0, None, 1e-5, 8, None, 0, None) == WS
    assert L.bl_forward_norm_grouped(3, None, 0, None, 1e-5, 8, A, 1 << 20, None) == INVALID
    wu = (ctypes.c_void_p * 3)(A, U, A)
    assert L.bl_forward_norm_grouped(3, arr, 0, wu, 1e-5, 8, A, 1 << 20, None) == ALIGN       # misaligned weight
    arr[2] = BLLinear(A, 1, 100, 64, A, A, A)
    assert L.bl_forward_norm_grouped(3, arr, 1, None, 1e-5, 8, A, 1 << 20, None) == SHAPE     # bad third problem
    assert L.bl_forward_norm_grouped(0, arr, 1, None, 1e-5, 8, None, 0, None) == OK


def test_grouped_host_validation(L):
    from bitlinear_bl_forward_b200.bl import BLLinear
    arr = (BLLinear * 3)()
    H = 0x7f0000001000          # host pointers are only copied from, never checked for alignment
    arr[0] = BLLinear(H, 1, 2560, 6912, A, A, H + 0x100000)
    arr[1] = BLLinear(H, 1, 2560, 6912, A, A, H + 0x200000)    # same X: staged once
    arr[2] = BLLinear(H + 0x300000, 1, 6912, 2560, A, A, H + 0x400000)
    need = L.bl_forward_grouped_host_staging_bytes(3, arr)
    # two distinct inputs and three outputs, none adjacent: five runs, 256-byte aligned each
    assert need == 2560 * 2 + 6912 * 2 + 6912 * 2 + 6912 * 2 + 2560 * 2
    # adjacent host regions share a run: X_a | X_b contiguous, outputs contiguous
    adj = (BLLinear * 3)()
    adj[0] = BLLinear(H, 1, 2560, 6912, A, A, H + 0x100000)
    adj[1] = BLLinear(H, 1, 2560, 6912, A, A, H + 0x100000 + 6912 * 2)
    adj[2] = BLLinear(H + 2560 * 2, 1, 6912, 2560, A, A, H + 0x100000 + 2 * 6912 * 2)
    in_run = 2560 * 2 + 6912 * 2                         # 18944 bytes -> 19200 with the run's alignment
    out_run = 2 * 6912 * 2 + 2560 * 2                    # 32768 bytes
    assert L.bl_forward_grouped_host_staging_bytes(3, adj) == (in_run + 255) // 256 * 256 + out_run
    # an output overlapping an input is rejected before any copy
    ov = (BLLinear * 1)()
    ov[0] = BLLinear(H, 1, 2560, 6912, A, A, H + 2048)
    assert L.bl_forward_grouped_host(1, ov, 8, A, 1 << 20, A, 1 << 20, None) == INVALID
    assert L.bl_forward_grouped_host_staging_bytes(9, arr) == 0
    assert L.bl_forward_grouped_host(3, arr, 8, None, 0, A, 1 << 20, None) == WS
    assert L.bl_forward_grouped_host(3, arr, 8, A, need - 1, A, 1 << 20, None) == WS
    assert L.bl_forward_grouped_host(3, arr, 8, U, need, A, 1 << 20, None) == ALIGN
    assert L.bl_forward_grouped_host(3, arr, 5, A, need, A, 1 << 20, None) == UNSUP
    assert L.bl_forward_grouped_host(9, arr, 8, A, need, A, 1 << 20, None) == UNSUP
    assert L.bl_forward_grouped_host(3, None, 8, A, need, A, 1 << 20, None) == INVALID
    arr[1] = BLLinear(H, 1, 2560, 6912, None, A, H + 0x200000)
    assert L.bl_forward_grouped_host(3, arr, 8, A, need, A, 1 << 20, None) == INVALID
    arr[1] = BLLinear(H, 1, 100, 6912, A, A, H + 0x200000)
    assert L.bl_forward_grouped_host_staging_bytes(3, arr) == 0
    assert L.bl_forward_grouped_host(3, arr, 8, A, need, A, 1 << 20, None) == SHAPE
    assert L.bl_forward_grouped_host(0, arr, 8, None, 0, None, 0, None) == OK
    arr[1] = BLLinear(H, 0, 2560, 6912, A, A, H + 0x200000)
    assert L.bl_forward_grouped_host(3, arr, 8, A, need, A, 1 << 20, None) == INVALID   # no empty problems


def test_grouped_host_graph_validation(L):
    # the recording entry validates like bl_forward_grouped_host before any
    # CUDA call, and clears the handle on error
    from bitlinear_bl_forward_b200.bl import BLLinear
    H = 0x7f0000001000
    ov = (BLLinear * 1)()
    ov[0] = BLLinear(H, 1, 2560, 6912, A, A, H + 2048)          # output overlaps the input
    h = ctypes.c_void_p(0x1234)
    assert L.bl_forward_grouped_host_graph(1, ov, 8, A, 1 << 20, A, 1 << 20, None, ctypes.byref(h)) == INVALID
    assert h.value is None
    h = ctypes.c_void_p(0x1234)
    assert L.bl_forward_grouped_host_graph(0, ov, 8, A, 1 << 20, A, 1 << 20, None, ctypes.byref(h)) == UNSUP
    assert h.value is None
    assert L.bl_forward_grouped_host_graph(9, ov, 8, A, 1 << 20, A, 1 << 20, None, ctypes.byref(h)) == UNSUP
    assert L.bl_forward_grouped_host_graph(1, None, 8, A, 1 << 20, A, 1 << 20, None, ctypes.byref(h)) == INVALID
    assert L.bl_forward_grouped_host_graph(1, ov, 8, A, 1 << 20, A, 1 << 20, None, None) == INVALID
    ok = (BLLinear * 1)()
    ok[0] = BLLinear(H, 1, 2560, 6912, A, A, H + 0x100000)
    assert L.bl_forward_grouped_host_graph(1, ok, 8, None, 0, A, 1 << 20, None, ctypes.byref(h)) == WS
    assert L.bl_forward_grouped_host_graph(1, ok, 5, A, 1 << 20, A, 1 << 20, None, ctypes.byref(h)) == UNSUP
    assert h.value is None
    assert L.bl_graph_launch(None, None) == INVALID
    L.bl_graph_destroy(None)   # a no-op


def test_base3_host_checks(L):
    # sizes: 4 * ceil(ceil(K / 20) / 4) bytes a row
    assert L.bl_packed_weight_bytes_b3(1, 64) == 16
    assert L.bl_packed_weight_bytes_b3(6912, 2560) == 6912 * 512
    assert L.bl_packed_weight_bytes_b3(28672, 8192) == 28672 * 1648
    assert L.bl_packed_weight_bytes_b3(4, 100) == 0                    # bad shape
    # one token only; K <= 8192; rejected before any launch
    assert L.bl_forward_b3(A, 2, 2560, 8, A, A, 8, A, None) == UNSUP
    assert L.bl_forward_b3(A, 1, 16384, 8, A, A, 8, A, None) == UNSUP
    assert L.bl_forward_b3(A, 1, 2560, 8, A, A, 5, A, None) == UNSUP     # bits
    assert L.bl_forward_b3(A, 1, 100, 8, A, A, 8, A, None) == SHAPE
    assert L.bl_forward_b3(None, 1, 2560, 8, A, A, 8, A, None) == INVALID
    assert L.bl_forward_b3(U, 1, 2560, 8, A, A, 8, A, None) == ALIGN
    assert L.bl_forward_b3(A, 0, 2560, 8, A, A, 8, A, None) == OK         # M == 0: no-op
    assert L.bl_matmul_i32_b3(A, 2, 2560, 8, A, A, None) == UNSUP
    assert L.bl_quantize_weights_b3(A, 8, 100, A, A, A, 1 << 12, None) == SHAPE
    assert L.bl_quantize_weights_b3(A, 8, 64, A, A, A, 0, None) == WS
    assert L.bl_unpack_weights_b3(U, 8, 64, A, None) == ALIGN


def test_probe_host_checks(L):
    assert L.bl_probe_mma_i8(0, 256, A, 148, None) == SHAPE
    assert L.bl_probe_mma_i8(16, 8, A, 148, None) == SHAPE
    assert L.bl_probe_mma_i8(16, 264, A, 148, None) == SHAPE
    assert L.bl_probe_mma_i8(16, 256, None, 148, None) == INVALID


def test_probe_pair_host_checks(L):
    assert L.bl_probe_mma_i8_pair(16, 128, A, 147, None) == SHAPE     # odd grid
    assert L.bl_probe_mma_i8_pair(16, 16, A, 148, None) == SHAPE      # n_cols % 32
    assert L.bl_probe_mma_i8_pair(16, 128, None, 148, None) == INVALID


def test_quant_act_packed4_host_checks(L):
    assert L.bl_quant_act_packed4(A, 4, 100, A, A, None) == SHAPE
    assert L.bl_quant_act_packed4(A, -1, 64, A, A, None) == SHAPE
    assert L.bl_quant_act_packed4(None, 4, 64, A, A, None) == INVALID
    assert L.bl_quant_act_packed4(A, 4, 64, U, A, None) == ALIGN
    assert L.bl_quant_act_packed4(A, 0, 64, A, A, None) == OK
