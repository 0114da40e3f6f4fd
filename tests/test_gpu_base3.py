"""GPU parity of the base-3 weight storage (five ternary weights a byte;
"BitNet b1.58: The 1-Bit Ternary LLM Architecture Guide", section "Why 1.58
Bits? The Power of Zero") against the CPU oracle.

Bars: gamma bitwise, stored bytes and unpacked codes byte-exact against
oracle.pack_base3 / the oracle's ternary codes, int32 accumulators exact,
bf16 outputs within 1 ulp of the oracle and bit-identical to bl_forward on the
2-bit storage of the same codes (same formulas and roundings).
"""

import numpy as np
import pytest
import torch

from bitlinear_bl_forward_b200 import bl
from bitlinear_bl_forward_b200.inputs import WORKLOADS, layer_inputs, random_case
from oracle import bitlinear_oracle as o
from tests.gpu_helpers import BF16_ULP_TOL, bf16_dev_to_bits, bf16_ulp_distance, x_to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bl.lib()
    bl.bl_device_status(clear=True)
    yield
    st, site = bl.bl_device_status(clear=True)
    assert st == 0, f"device status {st} at wait site {site}"


def check_b3(X, W, bits, full_oracle=True, sample_rows=None):
    N, K = W.shape
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wd = torch.from_numpy(W).cuda()
    Wp3, gd = bl.bl_quantize_weights_b3(Wd)
    Wp2, gd2 = bl.bl_quantize_weights(Wd)
    torch.cuda.synchronize()
    assert gd.cpu().numpy().view(np.uint32)[0] == np.float32(g).view(np.uint32)
    rows = np.arange(N) if sample_rows is None else np.asarray(sample_rows)
    assert np.array_equal(Wp3.cpu().numpy()[rows], o.pack_base3(c[rows]))
    assert np.array_equal(bl.bl_unpack_weights_b3(Wp3, N, K).cpu().numpy()[rows], c[rows])
    Xd = x_to_dev(X)
    q, s = o.act_quant(X, bits)
    acc = bl.bl_matmul_i32_b3(torch.from_numpy(q).cuda(), Wp3, N).cpu().numpy()
    Y3 = bl.bl_forward_b3(Xd, Wp3, gd, N, bits)
    Y2 = bl.bl_forward(Xd, Wp2, gd2, N, bits)
    torch.cuda.synchronize()
    assert torch.equal(Y3.view(torch.int16), Y2.view(torch.int16))
    if full_oracle:
        acc_o = o.matmul_i32(q, c)
        assert np.array_equal(acc, acc_o)
        Yo = o.round_to_bf16_bits(o.rescale(acc_o, g, s)[1])
        assert bf16_ulp_distance(bf16_dev_to_bits(Y3), Yo).max() <= BF16_ULP_TOL


@pytest.mark.parametrize("K,N", [(64, 7), (192, 33), (1536, 999), (2560, 6912), (3072, 130), (6912, 2560),
                                 (8192, 300), (8192, 20000)])
@pytest.mark.parametrize("bits", [8, 4])
def test_forward_b3_parity(K, N, bits):
    X, W = random_case(1, K, N, seed=900 + K + N + bits)
    check_b3(X, W, bits)


def test_forward_b3_layer_70b_full_size():
    # the 70B-class layer (K = 8192, N = 28672): big-ring mode; stored bytes
    # compared on a seeded sample of rows, outputs on every row
    w = WORKLOADS["layer_70b_m1"]
    X, W = layer_inputs(w, 0)
    rng = np.random.default_rng(3)
    check_b3(X, W, 8, full_oracle=True, sample_rows=np.sort(rng.choice(W.shape[0], 512, replace=False)))


def test_forward_b3_zero_token_and_back_to_back():
    X, W = random_case(1, 2560, 6912, seed=77)
    Wp3, g = bl.bl_quantize_weights_b3(torch.from_numpy(W).cuda())
    Z = torch.zeros((1, 2560), dtype=torch.bfloat16, device="cuda")
    Yz = bl.bl_forward_b3(Z, Wp3, g, 6912)
    assert torch.count_nonzero(Yz.float()).item() == 0
    Xd = x_to_dev(X)
    Y1 = bl.bl_forward_b3(Xd, Wp3, g, 6912)
    Y2 = torch.empty_like(Y1)
    for _ in range(3):
        bl.bl_forward_b3(Xd, Wp3, g, 6912, out=Y2)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
