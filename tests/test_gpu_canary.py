"""Out-of-bounds write checks: every output (and workspace) of the C ABI is
surrounded by guard bytes with a known pattern, which must be unchanged after
the call.  Shapes are ragged so that every kernel's tail handling is used
(decode kernels, the one-SM and CTA-pair tensor-core GEMMs with and without
the TMA-store epilogue, the quantisers, the weight packer)."""

import numpy as np
import pytest
import torch

from bitlinear_bl_forward_b200 import bl
from bitlinear_bl_forward_b200.inputs import random_case
from tests.gpu_helpers import x_to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps the 16-byte alignment of the body)
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bl.lib()
    bl.bl_device_status(clear=True)
    yield
    assert bl.bl_device_status(clear=True) == (0, 0)


class Guarded:
    """A device tensor of `shape`/`dtype` inside a guarded byte buffer."""

    def __init__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape) if nbytes else \
            torch.empty(shape, dtype=dtype, device="cuda")

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[-GUARD:].cpu().numpy()
        return bool(np.all(head == PATTERN) and np.all(tail == PATTERN))


FWD = [(1, 2560, 700), (1, 6912, 130), (1, 8192, 8200), (2, 192, 100), (3, 64, 129), (17, 320, 130),
       (64, 256, 72), (130, 256, 300), (130, 256, 304), (257, 192, 136)]


@pytest.mark.parametrize("M,K,N", FWD)
def test_forward_writes_stay_in_bounds(M, K, N):
    X, W = random_case(M, K, N, seed=M + K + N)
    Wp, g = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
    Y = Guarded((M, N), torch.bfloat16)
    need = bl.bl_forward_workspace_bytes(M, K, N)
    ws = Guarded((max(need, 16),), torch.uint8)
    bl.bl_forward(x_to_dev(X), Wp, g, N, out=Y.t, workspace=ws.t)
    assert Y.intact() and ws.intact()
    # the same through the variants
    Y2 = Guarded((M, N), torch.bfloat16)
    need2 = bl.bl_forward_ex_workspace_bytes(M, K, N, 8, 1)
    ws2 = Guarded((max(need2, 16),), torch.uint8)
    bias = torch.randn(N, device="cuda")
    bl.bl_forward_ex(x_to_dev(X), Wp, g, N, per_tensor=True, bias=bias, out=Y2.t, workspace=ws2.t)
    assert Y2.intact() and ws2.intact()
    Y3 = Guarded((M, N), torch.bfloat16)
    need3 = bl.bl_forward_relu2_workspace_bytes(M, K, N)
    ws3 = Guarded((max(need3, 16),), torch.uint8)
    bl.bl_forward_relu2(x_to_dev(X), x_to_dev(X), Wp, g, N, out=Y3.t, workspace=ws3.t)
    assert Y3.intact() and ws3.intact()
    Y4 = Guarded((M, N), torch.bfloat16)
    ws4 = Guarded((bl.bl_forward_rmsnorm_workspace_bytes(M, K, N),), torch.uint8)
    nw = torch.rand(K, device="cuda").to(torch.bfloat16)
    bl.bl_forward_rmsnorm(x_to_dev(X), Wp, g, N, norm_weight=nw, out=Y4.t, workspace=ws4.t)
    assert Y4.intact() and ws4.intact()
    Y5 = Guarded((M, N), torch.bfloat16)
    ws5 = Guarded((bl.bl_forward_layernorm_workspace_bytes(M, K, N),), torch.uint8)
    bl.bl_forward_layernorm(x_to_dev(X), Wp, g, N, out=Y5.t, workspace=ws5.t)
    assert Y5.intact() and ws5.intact()


def test_grouped_writes_stay_in_bounds():
    probs, outs = [], []
    for j, (K, N) in enumerate([(2560, 700), (2560, 33), (2048, 1000), (6912, 130)]):
        X, W = random_case(1, K, N, seed=40 + j)
        Wp, g = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs.append((x_to_dev(X), Wp, g, N))
        outs.append(Guarded((1, N), torch.bfloat16))
    bl.bl_forward_grouped(probs, outs=[o.t for o in outs])
    assert all(o.intact() for o in outs)
    for norm in (bl.BL_NORM_RMS, bl.BL_NORM_LAYER):
        outs = [Guarded((1, N), torch.bfloat16) for (_, _, _, N) in probs]
        nws = [torch.rand(X.shape[1], device="cuda").to(torch.bfloat16) for (X, _, _, _) in probs] \
            if norm == bl.BL_NORM_RMS else None
        bl.bl_forward_norm_grouped(probs, norm, nws, outs=[o.t for o in outs])
        assert all(o.intact() for o in outs)


@pytest.mark.parametrize("M,K", [(1, 64), (5, 192), (9, 6912), (3, 16384)])
def test_quantisers_write_in_bounds(M, K):
    X, _ = random_case(M, K, 8, seed=K)
    for bits in (8, 4):
        Xq = Guarded((M, K), torch.int8)
        s = Guarded((M,), torch.float32)
        bl.lib().bl_quant_act(x_to_dev(X).data_ptr(), M, K, bits, Xq.t.data_ptr(), s.t.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
        assert Xq.intact() and s.intact()
        Xr = Guarded((M, K), torch.int8)
        sr = Guarded((M,), torch.float32)
        bl.lib().bl_quant_act_relu2(x_to_dev(X).data_ptr(), None, M, K, bits, Xr.t.data_ptr(), sr.t.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
        assert Xr.intact() and sr.intact()
        Xn = Guarded((M, K), torch.int8)
        sn = Guarded((M,), torch.float32)
        ms = Guarded((M,), torch.float32)
        bl.lib().bl_quant_act_rmsnorm(x_to_dev(X).data_ptr(), None, 1e-5, M, K, bits, Xn.t.data_ptr(),
                                      sn.t.data_ptr(), ms.t.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert Xn.intact() and sn.intact() and ms.intact()
        Xl = Guarded((M, K), torch.int8)
        sl = Guarded((M,), torch.float32)
        mu = Guarded((M,), torch.float32)
        var = Guarded((M,), torch.float32)
        bl.lib().bl_quant_act_layernorm(x_to_dev(X).data_ptr(), 1e-5, M, K, bits, Xl.t.data_ptr(), sl.t.data_ptr(),
                                        mu.t.data_ptr(), var.t.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert Xl.intact() and sl.intact() and mu.intact() and var.intact()


@pytest.mark.parametrize("N,K", [(1, 64), (33, 192), (700, 2560), (130, 6912)])
def test_weight_packer_and_matmul_in_bounds(N, K):
    _, W = random_case(1, K, N, seed=N)
    Wd = torch.from_numpy(W).cuda()
    Wp = Guarded((N, K // 4), torch.uint8)
    g = Guarded((1,), torch.float32)
    wsn = int(bl.lib().bl_quantize_weights_workspace_bytes(N, K))
    ws = Guarded((wsn,), torch.uint8)
    st = bl.lib().bl_quantize_weights(Wd.data_ptr(), N, K, Wp.t.data_ptr(), g.t.data_ptr(), ws.t.data_ptr(), wsn,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0 and Wp.intact() and g.intact() and ws.intact()
    codes = Guarded((N, K), torch.int8)
    assert bl.lib().bl_unpack_weights(Wp.t.data_ptr(), N, K, codes.t.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream) == 0
    assert codes.intact()
    for M in (1, 3, 70):
        q = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda")
        acc = Guarded((M, N), torch.int32)
        wsm = int(bl.lib().bl_matmul_i32_workspace_bytes(M, K, N))
        wsg = Guarded((max(wsm, 16),), torch.uint8)
        assert bl.lib().bl_matmul_i32(q.data_ptr(), M, K, N, Wp.t.data_ptr(), acc.t.data_ptr(), wsg.t.data_ptr(),
                                      wsm, torch.cuda.current_stream().cuda_stream) == 0
        assert acc.intact() and wsg.intact()
