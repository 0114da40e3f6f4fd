"""Thin Python binding of libbitlinear (include/bitlinear.h).

Argument marshalling only: every function checks dtypes/devices, allocates
outputs and workspace with torch (device memory plumbing), passes raw device
pointers and torch's current CUDA stream to the C ABI, and raises BLError on a
non-OK status.  All arithmetic runs in the library's CUDA kernels; there is no
fallback of any kind -- if libbitlinear.so is missing the call fails.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGNMENT",
    4: "BL_ERR_UNSUPPORTED", 5: "BL_ERR_CUDA", 6: "BL_ERR_TIMEOUT", 7: "BL_ERR_WORKSPACE",
    8: "BL_ERR_SCRATCH_LIMIT",
}

# name -> (restype, argtypes), mirroring include/bitlinear.h
_i64, _sz, _p, _int = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "bl_status_string": (ctypes.c_char_p, [_int]),
    "bl_version": (_int, []),
    "bl_packed_weight_bytes": (_sz, [_i64, _i64]),
    "bl_quantize_weights_workspace_bytes": (_sz, [_i64, _i64]),
    "bl_quantize_weights": (_int, [_p, _i64, _i64, _p, _p, _p, _sz, _p]),
    "bl_unpack_weights": (_int, [_p, _i64, _i64, _p, _p]),
    "bl_quant_act": (_int, [_p, _i64, _i64, _int, _p, _p, _p]),
    "bl_quant_act_packed4": (_int, [_p, _i64, _i64, _p, _p, _p]),
    "bl_forward_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "bl_forward": (_int, [_p, _i64, _i64, _i64, _p, _p, _int, _p, _p, _sz, _p]),
    "bl_forward_f32": (_int, [_p, _i64, _i64, _i64, _p, _p, _int, _p, _p, _sz, _p]),
    "bl_forward_noalloc": (_int, [_p, _i64, _i64, _i64, _p, _p, _int, _p, _p]),
    "bl_forward_grouped_workspace_bytes": (_sz, [_int, _p, _int]),
    "bl_forward_grouped": (_int, [_int, _p, _int, _p, _sz, _p]),
    "bl_forward_relu2_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "bl_forward_relu2": (_int, [_p, _p, _i64, _i64, _i64, _p, _p, _int, _p, _p, _sz, _p]),
    "bl_quant_act_relu2": (_int, [_p, _p, _i64, _i64, _int, _p, _p, _p]),
    "bl_forward_ex_workspace_bytes": (_sz, [_i64, _i64, _i64, _int, ctypes.c_uint]),
    "bl_forward_ex": (_int, [_p, _i64, _i64, _i64, _p, _p, _int, ctypes.c_uint, _p, _p, _p, _sz, _p]),
    "bl_forward_rmsnorm_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "bl_forward_rmsnorm": (_int, [_p, _p, ctypes.c_float, _i64, _i64, _i64, _p, _p, _int, _p, _p, _sz, _p]),
    "bl_quant_act_rmsnorm": (_int, [_p, _p, ctypes.c_float, _i64, _i64, _int, _p, _p, _p, _p]),
    "bl_forward_layernorm_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "bl_forward_layernorm": (_int, [_p, ctypes.c_float, _i64, _i64, _i64, _p, _p, _int, _p, _p, _sz, _p]),
    "bl_quant_act_layernorm": (_int, [_p, ctypes.c_float, _i64, _i64, _int, _p, _p, _p, _p, _p]),
    "bl_forward_grouped_host_staging_bytes": (_sz, [_int, _p]),
    "bl_forward_grouped_host": (_int, [_int, _p, _int, _p, _sz, _p, _sz, _p]),
    "bl_forward_grouped_host_graph": (_int, [_int, _p, _int, _p, _sz, _p, _sz, _p, ctypes.POINTER(_p)]),
    "bl_graph_launch": (_int, [_p, _p]),
    "bl_graph_destroy": (None, [_p]),
    "bl_forward_norm_grouped_workspace_bytes": (_sz, [_int, _p, _int]),
    "bl_forward_norm_grouped": (_int, [_int, _p, _int, _p, ctypes.c_float, _int, _p, _sz, _p]),
    "bl_matmul_i32_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_matmul_i32": (_int, [_p, _i64, _i64, _i64, _p, _p, _p, _sz, _p]),
    "bl_device_status": (_int, [_int, ctypes.POINTER(_int)]),
    "bl_selftest_wait_timeout": (_int, [ctypes.c_ulonglong, _p, _p]),
    "bl_probe_mma_i8": (_int, [_int, _int, _p, _int, _p]),
    "bl_probe_mma_i8_pair": (_int, [_int, _int, _p, _int, _p]),
    "bl_packed_weight_bytes_b3": (_sz, [_i64, _i64]),
    "bl_quantize_weights_b3": (_int, [_p, _i64, _i64, _p, _p, _p, _sz, _p]),
    "bl_unpack_weights_b3": (_int, [_p, _i64, _i64, _p, _p]),
    "bl_forward_b3": (_int, [_p, _i64, _i64, _i64, _p, _p, _int, _p, _p]),
    "bl_matmul_i32_b3": (_int, [_p, _i64, _i64, _i64, _p, _p, _p]),
}

_lib = None


class BLLinear(ctypes.Structure):
    """Mirror of the C struct bl_linear (one problem of bl_forward_grouped)."""
    _fields_ = [("X", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64),
                ("Wp", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("Y", ctypes.c_void_p)]


class BLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({lib().bl_status_string(self.status).decode()})")


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so (built in-tree by bitlinear_bl_forward_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bitlinear_bl_forward_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(st: int, where: str):
    if st != BL_OK:
        raise BLError(st, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# C-ABI mirrors
# ---------------------------------------------------------------------------

def bl_packed_weight_bytes(N: int, K: int) -> int:
    return int(lib().bl_packed_weight_bytes(N, K))


def bl_quantize_weights(W: torch.Tensor):
    """fp32 [N, K] -> (packed uint8 [N, K/4], gamma fp32 [1])."""
    N, K = W.shape
    pW = _dev(W, torch.float32, "W")
    Wp = torch.empty((N, max(K // 4, 1)), dtype=torch.uint8, device=W.device)
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    ws = _workspace(int(lib().bl_quantize_weights_workspace_bytes(N, K)), W.device)
    _check(lib().bl_quantize_weights(pW, N, K, Wp.data_ptr(), gamma.data_ptr(),
                                     ws.data_ptr() if ws is not None else None,
                                     ws.numel() if ws is not None else 0, _stream()),
           "bl_quantize_weights")
    return Wp, gamma


def bl_unpack_weights(Wp: torch.Tensor, N: int, K: int) -> torch.Tensor:
    p = _dev(Wp, torch.uint8, "Wp")
    codes = torch.empty((N, K), dtype=torch.int8, device=Wp.device)
    _check(lib().bl_unpack_weights(p, N, K, codes.data_ptr(), _stream()), "bl_unpack_weights")
    return codes


def bl_quant_act(X: torch.Tensor, bits: int = 8):
    """bf16 [M, K] -> (int8 codes [M, K], scale fp32 [M])."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib().bl_quant_act(px, M, K, bits, Xq.data_ptr(), s.data_ptr(), _stream()), "bl_quant_act")
    return Xq, s


def bl_quant_act_packed4(X: torch.Tensor):
    """bf16 [M, K] -> (4-bit codes packed two a byte uint8 [M, K/2], scale fp32 [M])."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    Xq4 = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib().bl_quant_act_packed4(px, M, K, Xq4.data_ptr(), s.data_ptr(), _stream()), "bl_quant_act_packed4")
    return Xq4, s


def bl_forward_workspace_bytes(M: int, K: int, N: int, bits: int = 8) -> int:
    return int(lib().bl_forward_workspace_bytes(M, K, N, bits))


def bl_forward(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
               out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """BitLinear forward: bf16 [M, K] activations, packed weights -> bf16 [M, N]."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    need = bl_forward_workspace_bytes(M, K, N, bits)
    ws = workspace if workspace is not None else _workspace(need, X.device)
    _check(lib().bl_forward(px, M, K, N, pw, pg, bits, py,
                            ws.data_ptr() if ws is not None else None,
                            ws.numel() if ws is not None else 0, _stream()), "bl_forward")
    return Y


def bl_forward_f32(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8) -> torch.Tensor:
    """As bl_forward, fp32 output before the bf16 rounding (test export)."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    ws = _workspace(bl_forward_workspace_bytes(M, K, N, bits), X.device)
    _check(lib().bl_forward_f32(px, M, K, N, pw, pg, bits, Y.data_ptr(),
                                ws.data_ptr() if ws is not None else None,
                                ws.numel() if ws is not None else 0, _stream()), "bl_forward_f32")
    return Y


def bl_forward_noalloc(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """bl_forward without a workspace: for callers that cannot allocate device
    memory per call, the library keeps the scratch in a static device array
    (limits M*K <= 16 MiB, M <= 8192 when M > 2; calls that overlap on the GPU
    race on it).  Only the output buffer is passed in."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    _check(lib().bl_forward_noalloc(px, M, K, N, pw, pg, bits, py, _stream()), "bl_forward_noalloc")
    return Y


def _grouped_structs(problems, outs):
    arr = (BLLinear * max(1, len(problems)))()
    for i, ((X, Wp, gamma, N), Y) in enumerate(zip(problems, outs)):
        M, K = X.shape
        arr[i] = BLLinear(_dev(X, torch.bfloat16, "X"), M, K, N, _dev(Wp, torch.uint8, "Wp"),
                          _dev(gamma, torch.float32, "gamma"), _dev(Y, torch.bfloat16, "out"))
    return arr


def bl_forward_grouped_workspace_bytes(problems, bits: int = 8) -> int:
    """problems: list of (X, Wp, gamma, N)."""
    outs = [torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=X.device) for (X, _, _, N) in problems]
    arr = _grouped_structs(problems, outs)
    return int(lib().bl_forward_grouped_workspace_bytes(len(problems), arr, bits))


def bl_forward_grouped(problems, bits: int = 8, outs=None, workspace: torch.Tensor | None = None):
    """Several independent BitLinear forwards in one call (problems: list of
    (X bf16 [M, K], Wp, gamma, N)); returns the list of bf16 outputs."""
    if outs is None:
        outs = [torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=X.device) for (X, _, _, N) in problems]
    arr = _grouped_structs(problems, outs)
    ws = workspace
    if ws is None:
        need = int(lib().bl_forward_grouped_workspace_bytes(len(problems), arr, bits))
        ws = _workspace(need, problems[0][0].device if problems else "cuda")
    _check(lib().bl_forward_grouped(len(problems), arr, bits, ws.data_ptr() if ws is not None else None,
                                    ws.numel() if ws is not None else 0, _stream()), "bl_forward_grouped")
    return outs


class PreparedGrouped:
    """A bl_forward_grouped call whose arguments are checked and packed once
    (the bl_linear array, the workspace pointer): calling it issues the same
    C call on the current stream with no per-call marshalling.  The tensors
    must stay alive and in place; their contents may change between calls."""

    def __init__(self, problems, bits: int = 8, outs=None, workspace: torch.Tensor | None = None):
        if outs is None:
            outs = [torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=X.device) for (X, _, _, N) in problems]
        self.outs = outs
        self._keep = (list(problems), list(outs), workspace)
        self._n = len(problems)
        self._arr = _grouped_structs(problems, outs)
        self._bits = bits
        ws = workspace
        if ws is None:
            need = int(lib().bl_forward_grouped_workspace_bytes(self._n, self._arr, bits))
            ws = _workspace(need, problems[0][0].device if problems else "cuda")
            self._keep = self._keep + (ws,)
        self._wsp = ws.data_ptr() if ws is not None else None
        self._wsn = ws.numel() if ws is not None else 0
        self._fn = lib().bl_forward_grouped

    def __call__(self):
        _check(self._fn(self._n, self._arr, self._bits, self._wsp, self._wsn, _stream()), "bl_forward_grouped")
        return self.outs


def _host(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def bl_forward_grouped_host_staging_bytes(problems, outs) -> int:
    """problems: list of (X host bf16 [M, K], Wp, gamma, N); outs: host bf16 [M, N]."""
    arr = _host_structs(problems, outs)
    return int(lib().bl_forward_grouped_host_staging_bytes(len(problems), arr))


def _host_structs(problems, outs):
    arr = (BLLinear * max(1, len(problems)))()
    for i, ((X, Wp, gamma, N), Y) in enumerate(zip(problems, outs)):
        M, K = X.shape
        if tuple(Y.shape) != (M, N):
            raise ValueError("output must be [M, N]")
        arr[i] = BLLinear(_host(X, torch.bfloat16, "X"), M, K, N, _dev(Wp, torch.uint8, "Wp"),
                          _dev(gamma, torch.float32, "gamma"), _host(Y, torch.bfloat16, "out"))
    return arr


class PreparedGroupedHost:
    """bl_forward_grouped_host prepared once: problems is a list of
    (X host bf16 [M, K], Wp, gamma, N) and outs the host bf16 [M, N] outputs
    (pinned memory keeps the copies asynchronous).  Each call enqueues on the
    current stream the input copies, the grouped forward and the output
    copies; synchronise the stream before reading the outputs.  graph=True
    records the call once as a CUDA graph (bl_forward_grouped_host_graph:
    this runs the step once on the current stream and waits for it) and each
    call replays it (bl_graph_launch), reading the current contents of the
    same host inputs."""

    def __init__(self, problems, outs, bits: int = 8, device="cuda", graph: bool = False):
        self.outs = outs
        self._n = len(problems)
        self._arr = _host_structs(problems, outs)
        self._bits = bits
        nst = int(lib().bl_forward_grouped_host_staging_bytes(self._n, self._arr))
        if nst == 0:
            raise ValueError("bad problem shapes")
        self._stg = torch.empty(nst, dtype=torch.uint8, device=device)
        nws = int(lib().bl_forward_grouped_workspace_bytes(self._n, self._arr, bits))
        self._ws = torch.empty(nws, dtype=torch.uint8, device=device) if nws else None
        self._keep = (list(problems), list(outs))
        self._args = (self._stg.data_ptr(), nst, self._ws.data_ptr() if self._ws is not None else None, nws)
        self._fn = lib().bl_forward_grouped_host
        self._graph = bl_forward_grouped_host_graph(self._n, self._arr, bits, *self._args) if graph else None

    def __call__(self):
        if self._graph is not None:
            bl_graph_launch(self._graph)
        else:
            _check(self._fn(self._n, self._arr, self._bits, *self._args, _stream()), "bl_forward_grouped_host")
        return self.outs

    def __del__(self):
        g = getattr(self, "_graph", None)
        if g is not None and _lib is not None:
            try:
                torch.cuda.synchronize()   # no replay may still be running when the graph is freed
            except Exception:
                pass
            bl_graph_destroy(g)
            self._graph = None


def bl_forward_grouped_host_graph(count, structs, bits, staging, staging_bytes, workspace, workspace_bytes):
    """Record a host-buffer grouped forward as a CUDA graph (returns the
    handle; see PreparedGroupedHost, which owns one)."""
    h = ctypes.c_void_p(None)
    _check(lib().bl_forward_grouped_host_graph(count, structs, bits, staging, staging_bytes, workspace,
                                               workspace_bytes, _stream(), ctypes.byref(h)),
           "bl_forward_grouped_host_graph")
    return h


def bl_graph_launch(graph):
    """One replay of a recorded graph on the current stream."""
    _check(lib().bl_graph_launch(graph, _stream()), "bl_graph_launch")


def bl_graph_destroy(graph):
    lib().bl_graph_destroy(graph)


def bl_forward_grouped_host(problems, outs, bits: int = 8):
    """One grouped forward on host-resident activations (see PreparedGroupedHost,
    which keeps its staging and workspace across calls); synchronises the
    stream before returning the host outputs."""
    PreparedGroupedHost(problems, outs, bits)()
    torch.cuda.current_stream().synchronize()
    return outs


def bl_forward_relu2_workspace_bytes(M: int, K: int, N: int, bits: int = 8) -> int:
    return int(lib().bl_forward_relu2_workspace_bytes(M, K, N, bits))


def bl_forward_relu2(G: torch.Tensor, U: torch.Tensor | None, Wp: torch.Tensor, gamma: torch.Tensor, N: int,
                     bits: int = 8, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Down projection of the squared-ReLU feed-forward: input max(0, G)^2
    (times U when given), bf16 [M, K] each -> bf16 [M, N]."""
    M, K = G.shape
    pg_in = _dev(G, torch.bfloat16, "G")
    pu = _dev(U, torch.bfloat16, "U") if U is not None else None
    if U is not None and tuple(U.shape) != (M, K):
        raise ValueError("U must have the shape of G")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=G.device)
    py = _dev(Y, torch.bfloat16, "out")
    ws = workspace
    if ws is None:
        ws = _workspace(bl_forward_relu2_workspace_bytes(M, K, N, bits), G.device)
    _check(lib().bl_forward_relu2(pg_in, pu, M, K, N, pw, pg, bits, py,
                                  ws.data_ptr() if ws is not None else None,
                                  ws.numel() if ws is not None else 0, _stream()), "bl_forward_relu2")
    return Y


def bl_quant_act_relu2(G: torch.Tensor, U: torch.Tensor | None, bits: int = 8):
    """max(0, G)^2 (times U) quantised per token -> (int8 codes [M, K], scale fp32 [M])."""
    M, K = G.shape
    pg_in = _dev(G, torch.bfloat16, "G")
    pu = _dev(U, torch.bfloat16, "U") if U is not None else None
    Xq = torch.empty((M, K), dtype=torch.int8, device=G.device)
    s = torch.empty(M, dtype=torch.float32, device=G.device)
    _check(lib().bl_quant_act_relu2(pg_in, pu, M, K, bits, Xq.data_ptr(), s.data_ptr(), _stream()),
           "bl_quant_act_relu2")
    return Xq, s


BL_ACT_PER_TENSOR = 1


def bl_forward_ex_workspace_bytes(M: int, K: int, N: int, bits: int = 8, flags: int = 0) -> int:
    return int(lib().bl_forward_ex_workspace_bytes(M, K, N, bits, flags))


def bl_forward_ex(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
                  per_tensor: bool = False, bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """bl_forward with the per-tensor activation scale and/or an fp32 bias [N]."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    pb = _dev(bias, torch.float32, "bias") if bias is not None else None
    flags = BL_ACT_PER_TENSOR if per_tensor else 0
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    ws = workspace
    if ws is None:
        ws = _workspace(bl_forward_ex_workspace_bytes(M, K, N, bits, flags), X.device)
    _check(lib().bl_forward_ex(px, M, K, N, pw, pg, bits, flags, pb, py,
                               ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0, _stream()), "bl_forward_ex")
    return Y


def bl_forward_rmsnorm_workspace_bytes(M: int, K: int, N: int, bits: int = 8) -> int:
    return int(lib().bl_forward_rmsnorm_workspace_bytes(M, K, N, bits))


def bl_forward_rmsnorm(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
                       norm_weight: torch.Tensor | None = None, eps: float = 1e-5,
                       out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """bl_forward on RMSNorm(X) (optional bf16 weight [K]), formed in the same
    kernels: bf16 [M, K] -> bf16 [M, N]."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pn = _dev(norm_weight, torch.bfloat16, "norm_weight") if norm_weight is not None else None
    if norm_weight is not None and tuple(norm_weight.shape) != (K,):
        raise ValueError("norm_weight must be [K]")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    ws = workspace
    if ws is None:
        ws = _workspace(bl_forward_rmsnorm_workspace_bytes(M, K, N, bits), X.device)
    _check(lib().bl_forward_rmsnorm(px, pn, eps, M, K, N, pw, pg, bits, py,
                                    ws.data_ptr() if ws is not None else None,
                                    ws.numel() if ws is not None else 0, _stream()), "bl_forward_rmsnorm")
    return Y


def bl_quant_act_rmsnorm(X: torch.Tensor, bits: int = 8, norm_weight: torch.Tensor | None = None,
                         eps: float = 1e-5):
    """RMSNorm(X) quantised per token -> (int8 codes [M, K], scale fp32 [M],
    mean of squares fp32 [M])."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pn = _dev(norm_weight, torch.bfloat16, "norm_weight") if norm_weight is not None else None
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    ms = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib().bl_quant_act_rmsnorm(px, pn, eps, M, K, bits, Xq.data_ptr(), s.data_ptr(), ms.data_ptr(),
                                      _stream()), "bl_quant_act_rmsnorm")
    return Xq, s, ms


BL_NORM_RMS = 0
BL_NORM_LAYER = 1


def bl_forward_layernorm_workspace_bytes(M: int, K: int, N: int, bits: int = 8) -> int:
    return int(lib().bl_forward_layernorm_workspace_bytes(M, K, N, bits))


def bl_forward_layernorm(X: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
                         eps: float = 1e-5, out: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None) -> torch.Tensor:
    """bl_forward on LayerNorm(X) (no affine parameters), formed in the same
    kernels: bf16 [M, K] -> bf16 [M, N]."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp, torch.uint8, "Wp")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    ws = workspace
    if ws is None:
        ws = _workspace(bl_forward_layernorm_workspace_bytes(M, K, N, bits), X.device)
    _check(lib().bl_forward_layernorm(px, eps, M, K, N, pw, pg, bits, py,
                                      ws.data_ptr() if ws is not None else None,
                                      ws.numel() if ws is not None else 0, _stream()), "bl_forward_layernorm")
    return Y


def bl_quant_act_layernorm(X: torch.Tensor, bits: int = 8, eps: float = 1e-5):
    """LayerNorm(X) quantised per token -> (int8 codes [M, K], scale fp32 [M],
    mean fp32 [M], variance fp32 [M])."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    mu = torch.empty(M, dtype=torch.float32, device=X.device)
    var = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib().bl_quant_act_layernorm(px, eps, M, K, bits, Xq.data_ptr(), s.data_ptr(), mu.data_ptr(),
                                        var.data_ptr(), _stream()), "bl_quant_act_layernorm")
    return Xq, s, mu, var


def bl_forward_norm_grouped_workspace_bytes(problems, bits: int = 8) -> int:
    """problems: list of (X, Wp, gamma, N)."""
    outs = [torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=X.device) for (X, _, _, N) in problems]
    arr = _grouped_structs(problems, outs)
    return int(lib().bl_forward_norm_grouped_workspace_bytes(len(problems), arr, bits))


def bl_forward_norm_grouped(problems, norm: int, norm_weights=None, eps: float = 1e-5, bits: int = 8, outs=None,
                            workspace: torch.Tensor | None = None):
    """Several normalised BitLinear forwards in one call (problems: list of
    (X bf16 [M, K], Wp, gamma, N); norm BL_NORM_RMS with optional per-problem
    bf16 weights, or BL_NORM_LAYER); returns the list of bf16 outputs."""
    if outs is None:
        outs = [torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=X.device) for (X, _, _, N) in problems]
    arr = _grouped_structs(problems, outs)
    wa = None
    if norm_weights is not None:
        ptrs = []
        for (X, _, _, _), w in zip(problems, norm_weights):
            if w is not None and tuple(w.shape) != (X.shape[1],):
                raise ValueError("norm weight must be [K]")
            ptrs.append(_dev(w, torch.bfloat16, "norm_weight") if w is not None else None)
        wa = (ctypes.c_void_p * len(ptrs))(*ptrs)
    ws = workspace
    if ws is None:
        need = int(lib().bl_forward_norm_grouped_workspace_bytes(len(problems), arr, bits))
        ws = _workspace(need, problems[0][0].device if problems else "cuda")
    _check(lib().bl_forward_norm_grouped(len(problems), arr, norm, wa, eps, bits,
                                         ws.data_ptr() if ws is not None else None,
                                         ws.numel() if ws is not None else 0, _stream()),
           "bl_forward_norm_grouped")
    return outs


def bl_matmul_i32(Xq: torch.Tensor, Wp: torch.Tensor, N: int) -> torch.Tensor:
    """Exact int32 accumulators of int8 [M, K] codes x packed weights (test export)."""
    M, K = Xq.shape
    px = _dev(Xq, torch.int8, "Xq")
    pw = _dev(Wp, torch.uint8, "Wp")
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    ws = _workspace(int(lib().bl_matmul_i32_workspace_bytes(M, K, N)), Xq.device)
    _check(lib().bl_matmul_i32(px, M, K, N, pw, acc.data_ptr(),
                               ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0, _stream()), "bl_matmul_i32")
    return acc


def bl_device_status(clear: bool = True):
    """(status, site) recorded by kernels since the last clear."""
    site = ctypes.c_int(0)
    st = lib().bl_device_status(1 if clear else 0, ctypes.byref(site))
    return int(st), int(site.value)


def bl_selftest_wait_timeout(limit_ns: int) -> torch.Tensor:
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(lib().bl_selftest_wait_timeout(limit_ns, out.data_ptr(), _stream()), "bl_selftest_wait_timeout")
    return out


def bl_probe_mma_i8(n_mma: int, n_cols: int = 256, grid: int | None = None) -> torch.Tensor:
    """tcgen05 kind::i8 rate probe: int64 [grid, 2] of (SM cycles, ns) per CTA
    for n_mma MMAs of 128 x n_cols x 32 (one CTA per SM by default)."""
    if grid is None:
        grid = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    out = torch.zeros((grid, 2), dtype=torch.int64, device="cuda")
    _check(lib().bl_probe_mma_i8(n_mma, n_cols, out.data_ptr(), grid, _stream()), "bl_probe_mma_i8")
    return out


# ---------------------------------------------------------------------------
# base-3 weight storage (five weights a byte)
# ---------------------------------------------------------------------------

def bl_packed_weight_bytes_b3(N: int, K: int) -> int:
    return int(lib().bl_packed_weight_bytes_b3(N, K))


def bl_quantize_weights_b3(W: torch.Tensor):
    """fp32 [N, K] -> (base-3 uint8 [N, row bytes], gamma fp32 [1])."""
    N, K = W.shape
    pW = _dev(W, torch.float32, "W")
    nb = bl_packed_weight_bytes_b3(N, K)
    Wp3 = torch.empty((N, max(nb // max(N, 1), 1)), dtype=torch.uint8, device=W.device)
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    ws = _workspace(int(lib().bl_quantize_weights_workspace_bytes(N, K)), W.device)
    _check(lib().bl_quantize_weights_b3(pW, N, K, Wp3.data_ptr(), gamma.data_ptr(),
                                        ws.data_ptr() if ws is not None else None,
                                        ws.numel() if ws is not None else 0, _stream()), "bl_quantize_weights_b3")
    return Wp3, gamma


def bl_unpack_weights_b3(Wp3: torch.Tensor, N: int, K: int) -> torch.Tensor:
    p = _dev(Wp3, torch.uint8, "Wp3")
    codes = torch.empty((N, K), dtype=torch.int8, device=Wp3.device)
    _check(lib().bl_unpack_weights_b3(p, N, K, codes.data_ptr(), _stream()), "bl_unpack_weights_b3")
    return codes


def bl_forward_b3(X: torch.Tensor, Wp3: torch.Tensor, gamma: torch.Tensor, N: int, bits: int = 8,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """One-token BitLinear forward on base-3 weights: bf16 [1, K] -> bf16 [1, N]."""
    M, K = X.shape
    px = _dev(X, torch.bfloat16, "X")
    pw = _dev(Wp3, torch.uint8, "Wp3")
    pg = _dev(gamma, torch.float32, "gamma")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    py = _dev(Y, torch.bfloat16, "out")
    _check(lib().bl_forward_b3(px, M, K, N, pw, pg, bits, py, _stream()), "bl_forward_b3")
    return Y


def bl_matmul_i32_b3(Xq: torch.Tensor, Wp3: torch.Tensor, N: int) -> torch.Tensor:
    """Exact int32 accumulators of one token's int8 codes x base-3 weights (test export)."""
    M, K = Xq.shape
    px = _dev(Xq, torch.int8, "Xq")
    pw = _dev(Wp3, torch.uint8, "Wp3")
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _check(lib().bl_matmul_i32_b3(px, M, K, N, pw, acc.data_ptr(), _stream()), "bl_matmul_i32_b3")
    return acc


def bl_probe_mma_i8_pair(n_mma: int, n_cols: int = 128, grid: int | None = None) -> torch.Tensor:
    """CTA-pair (cta_group::2) kind::i8 rate probe: int64 [grid, 2] of (SM
    cycles, ns) per CTA for n_mma MMAs of 256 x n_cols x 32 over each pair."""
    if grid is None:
        grid = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count // 2 * 2
    out = torch.zeros((grid, 2), dtype=torch.int64, device="cuda")
    _check(lib().bl_probe_mma_i8_pair(n_mma, n_cols, out.data_ptr(), grid, _stream()), "bl_probe_mma_i8_pair")
    return out
