"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle.

Bars: bit-exact gamma, packed bytes, ternary codes, int8/int4 activation codes,
activation scales and int32 accumulators; fp32 rescaled outputs within 1e-3
relative of the oracle; bf16 outputs within 1 ulp of the oracle's fp32 value
rounded to bf16.  Inputs are the seeded synthetic workloads; the oracle never
sees a value produced by the GPU.
"""

import functools

import numpy as np
import pytest
import torch

from bitlinear_bl_forward_b200 import bl
from bitlinear_bl_forward_b200.inputs import WORKLOADS, layer_inputs, make_weight, random_case
from oracle import bitlinear_oracle as o
from tests.gpu_helpers import (BF16_ULP_TOL, F32_REL_TOL, bf16_dev_to_bits, bf16_ulp_distance, rel_err,
                               x_to_dev)

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


@functools.lru_cache(maxsize=8)
def oracle_weights(key):
    """(W, gamma, codes, packed) for a cached weight (key = workload, layer)."""
    name, i = key
    _, W = layer_inputs(WORKLOADS[name], i, M=1)
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    return W, g, c, o.pack_ternary(c)


def check_weights(W, g, codes, packed):
    N, K = W.shape
    Wd = torch.from_numpy(W).cuda()
    Wp, gd = bl.bl_quantize_weights(Wd)
    torch.cuda.synchronize()
    assert gd.cpu().numpy().view(np.uint32)[0] == np.float32(g).view(np.uint32), (gd.item(), g)
    assert np.array_equal(Wp.cpu().numpy(), packed)
    cd = bl.bl_unpack_weights(Wp, N, K).cpu().numpy()
    assert np.array_equal(cd, codes)
    return Wp, gd


def check_act(x_bits, bits):
    q, s = o.act_quant(x_bits, bits)
    qd, sd = bl.bl_quant_act(x_to_dev(x_bits), bits)
    assert np.array_equal(qd.cpu().numpy(), q)
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s.view(np.uint32))
    return q, s


def check_forward(x_bits, Wp, g, codes, bits, rows=None):
    """Compare bl_forward / bl_forward_f32 / bl_matmul_i32 with the oracle;
    `rows` restricts the oracle to a sample of tokens (per-token quantisation
    makes each token independent)."""
    N = codes.shape[0]
    Xd = x_to_dev(x_bits)
    q_full, s_full = o.act_quant(x_bits, bits)
    sel = np.arange(x_bits.shape[0]) if rows is None else np.asarray(rows)
    q, s = q_full[sel], s_full[sel]
    acc = o.matmul_i32(q, codes)
    y64, y32 = o.rescale(acc, g, s)
    Y = o.round_to_bf16_bits(y32)

    accd = bl.bl_matmul_i32(torch.from_numpy(q_full).cuda(), Wp, N).cpu().numpy()[sel]
    assert np.array_equal(accd, acc)

    Yd = bf16_dev_to_bits(bl.bl_forward(Xd, Wp, torch.tensor([g], device="cuda"), N, bits))[sel]
    d = bf16_ulp_distance(Yd, Y)
    assert d.max() <= BF16_ULP_TOL, f"bf16 ulp distance {d.max()}"

    Yf = bl.bl_forward_f32(Xd, Wp, torch.tensor([g], device="cuda"), N, bits).cpu().numpy()[sel]
    e = rel_err(Yf, y64)
    assert e.max() <= F32_REL_TOL, f"fp32 rel err {e.max()}"
    # the kernels evaluate exactly the oracle's fp32 expression
    return float(np.mean(Yf.view(np.uint32) == y32.view(np.uint32))), float(np.mean(d == 0))


# ---------------------------------------------------------------------------
# failure path: bounded waits
# ---------------------------------------------------------------------------

def test_bounded_wait_times_out_cleanly():
    bl.bl_device_status(clear=True)
    out = bl.bl_selftest_wait_timeout(10_000_000)   # 10 ms
    st, site = bl.bl_device_status(clear=True)
    assert int(out.item()) == 0
    assert st == 6 and site == 0xEE
    # the context is still usable and the status word was cleared
    assert bl.bl_device_status(clear=True) == (0, 0)
    torch.ones(4, device="cuda").sum().item()


# ---------------------------------------------------------------------------
# small and ragged shapes
# ---------------------------------------------------------------------------

SMALL = [(1, 64, 1), (1, 256, 512), (2, 192, 100), (3, 64, 129), (16, 256, 512), (17, 320, 130),
         (33, 128, 257), (64, 256, 64), (100, 384, 300), (130, 256, 512), (257, 192, 129), (300, 1024, 700)]


@pytest.mark.parametrize("M,K,N", SMALL)
@pytest.mark.parametrize("bits", [8, 4])
def test_small_shapes(M, K, N, bits):
    X, W = random_case(M, K, N, seed=M * 1000 + K + N)
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, gd = check_weights(W, g, c, o.pack_ternary(c))
    check_act(X, bits)
    check_forward(X, Wp, g, c, bits)


# few weight-row tiles and long K (the one-SM GEMM with few tiles per launch)
SPLIT_K = [(16, 6912, 2560), (5, 4096, 300), (33, 2560, 1000), (64, 8192, 700), (3, 1024, 64)]


@pytest.mark.parametrize("M,K,N", SPLIT_K)
def test_few_tiles_long_k(M, K, N):
    X, W = random_case(M, K, N, seed=M * 100 + K + N)
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, gd = check_weights(W, g, c, o.pack_ternary(c))
    check_forward(X, Wp, g, c, 8)


# One-token shapes that reach each path of the row-lane decode kernel: rows
# that overflow the shared ring (K = 8192, 47-48 rows a CTA: chunks taken one
# at a time), more than 512 rows a CTA (the column-split fallback), rows of an
# odd number of 16-byte columns (the wider padding) with a partial last item,
# and fewer rows than CTAs.
ROW_LANE = [(8192, 7000, 8), (64, 80000, 8), (192, 5000, 4), (320, 33, 8), (6912, 2561, 8)]


@pytest.mark.parametrize("K,N,bits", ROW_LANE)
def test_decode_row_lane_paths(K, N, bits):
    X, W = random_case(1, K, N, seed=K + N)
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, gd = check_weights(W, g, c, o.pack_ternary(c))
    check_act(X, bits)
    check_forward(X, Wp, g, c, bits)


def test_zero_inputs_and_degenerate_rows():
    M, K, N = 5, 128, 96
    X, W = random_case(M, K, N, seed=7)
    X[1] = 0                       # all-zero token -> zero codes, zero output
    X[3, :] = X[3, 0]              # constant row
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, _ = check_weights(W, g, c, o.pack_ternary(c))
    check_act(X, 8)
    check_forward(X, Wp, g, c, 8)
    # all-zero weights: gamma = 1e-5, codes 0
    Wz = np.zeros((N, K), np.float32)
    gz = o.absmean_scale(Wz)
    cz = o.ternary_codes(Wz, gz)
    Wpz, _ = check_weights(Wz, gz, cz, o.pack_ternary(cz))
    check_forward(X, Wpz, gz, cz, 8)


def test_exact_ties_in_weights_and_activations():
    # weights at exactly +-gamma/2 and +-3gamma/2, activations with x*s exact .5
    K, N = 64, 16
    W = np.zeros((N, K), np.float32)
    W[:, ::4] = 0.25
    W[:, 1::4] = -0.25
    W[:, 2::4] = 0.0625
    W[:, 3::4] = -0.1875
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, _ = check_weights(W, g, c, o.pack_ternary(c))
    xf = np.zeros((3, K), np.float32)
    xf[:, 0] = 127.0
    xf[0, 1:8] = [2.5, 3.5, -0.5, -1.5, 0.5, 126.5, -126.5]
    xf[1, 0] = 3.0
    xf[1, 1:4] = [1.5, -1.5, 0.75]   # s = f32(127/3): 1.5*s is an fp32 tie -> 64
    xf[2, 0] = 7.0
    xf[2, 1:5] = [3.5, -3.5, 2.5, 0.5]
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    for bits in (8, 4):
        q, _ = check_act(xb, bits)
        check_forward(xb, Wp, g, c, bits)
    q8, _ = o.act_quant(xb, 8)
    assert q8[1, 1] == 64


def test_m_zero_is_a_noop():
    N, K = 32, 64
    Wp = torch.zeros((N, K // 4), dtype=torch.uint8, device="cuda")
    X = torch.zeros((0, K), dtype=torch.bfloat16, device="cuda")
    Y = bl.bl_forward(X, Wp, torch.ones(1, device="cuda"), N)
    assert Y.shape == (0, N)


def test_gemv_and_tensor_core_paths_agree():
    # M = 2 runs the decode kernel, M = 3 the tensor-core kernel; token rows
    # are independent, so the shared rows must match bit for bit.
    X, W = random_case(3, 2560, 700, seed=11)
    g = o.absmean_scale(W)
    c = o.ternary_codes(W, g)
    Wp, gd = check_weights(W, g, c, o.pack_ternary(c))
    y2 = bl.bl_forward_f32(x_to_dev(X[:2]), Wp, gd, 700).cpu().numpy()
    y3 = bl.bl_forward_f32(x_to_dev(X), Wp, gd, 700).cpu().numpy()
    assert np.array_equal(y2.view(np.uint32), y3[:2].view(np.uint32))


def test_streams_are_respected():
    # two independent problems on two streams give the same results as serial runs
    X, W = random_case(40, 512, 384, seed=12)
    Wd = torch.from_numpy(W).cuda()
    Wp, gd = bl.bl_quantize_weights(Wd)
    Xd = x_to_dev(X)
    ref = bl.bl_forward(Xd, Wp, gd, 384).clone()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        a = bl.bl_forward(Xd, Wp, gd, 384)
    with torch.cuda.stream(s2):
        b = bl.bl_forward(Xd[:1].contiguous(), Wp, gd, 384)
    torch.cuda.synchronize()
    assert torch.equal(a, ref) and torch.equal(b[0], ref[0])


# ---------------------------------------------------------------------------
# the workloads at full size
# ---------------------------------------------------------------------------

def run_workload(name, rows=None):
    w = WORKLOADS[name]
    for i, L in enumerate(w.layers):
        X, _ = layer_inputs(w, i)
        W, g, c, p = oracle_weights((name if not name.startswith("layer_70b") else "layer_70b_m1", i))
        Wp, gd = check_weights(W, g, c, p)
        check_act(X, w.bits)
        exact32, exact16 = check_forward(X, Wp, g, c, w.bits, rows=rows)
        print(f"{name}/{L.name}: fp32 bitwise-equal {exact32:.6f}, bf16 equal {exact16:.6f}")


def test_workload_tiny():
    run_workload("tiny")


def test_workload_decode_2b():
    run_workload("decode_2b")


def test_workload_prefill_2b():
    run_workload("prefill_2b")


@pytest.mark.parametrize("name", ["layer_70b_m1", "layer_70b_m16", "layer_70b_m128"])
def test_workload_70b(name):
    run_workload(name)


def test_workload_70b_m2048_sampled():
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(2048, 64, replace=False))
    run_workload("layer_70b_m2048", rows=rows)


def test_workload_a48():
    run_workload("a48")


# ---------------------------------------------------------------------------
# grouped forward
# ---------------------------------------------------------------------------

def oracle_bf16(x_bits, codes, g, bits=8):
    q, s = o.act_quant(x_bits, bits)
    return o.round_to_bf16_bits(o.rescale(o.matmul_i32(q, codes), g, s)[1])


def test_grouped_decode_matches_single_calls_and_oracle():
    # the 2B decode step in one launch: up and gate share X (K = 2560), down
    # reads its own input (K = 6912)
    w = WORKLOADS["decode_2b"]
    probs, refs = [], []
    xs = {}
    for i, L in enumerate(w.layers):
        X, _ = layer_inputs(w, i)
        key = L.x_layer if L.x_layer >= 0 else i
        if key not in xs:
            xs[key] = x_to_dev(X)
        Xd = xs[key]
        W, g, c, p = oracle_weights(("decode_2b", i))
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        N = W.shape[0]
        probs.append((Xd, Wp, gd, N))
        refs.append((bl.bl_forward(Xd, Wp, gd, N), oracle_bf16(X, c, g)))
    outs = bl.bl_forward_grouped(probs)
    torch.cuda.synchronize()
    for Yg, (Ys, Yo) in zip(outs, refs):
        assert torch.equal(Yg, Ys)
        assert bf16_ulp_distance(bf16_dev_to_bits(Yg), Yo).max() <= BF16_ULP_TOL
    # the same group twice more in a row, outputs reused (back-to-back launches)
    for _ in range(2):
        bl.bl_forward_grouped(probs, outs=outs)
    torch.cuda.synchronize()
    for Yg, (Ys, _) in zip(outs, refs):
        assert torch.equal(Yg, Ys)


def test_grouped_decode_mixed_k_one_launch():
    # eight one-token problems of eight different K in one launch: one register
    # width class, the rest on the shared-memory path; ragged row counts
    # (including one row, fewer rows than CTAs, and rows that do not fill a
    # row group), bits 8 and 4
    shapes = [(64, 7), (512, 1), (1536, 999), (2560, 6912), (3072, 130), (4096, 2049), (6912, 2560), (8192, 3)]
    for bits in (8, 4):
        probs, cases = [], []
        for j, (K, N) in enumerate(shapes):
            X, W = random_case(1, K, N, seed=500 + j + 10 * bits)
            g = o.absmean_scale(W)
            c = o.ternary_codes(W, g)
            Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
            probs.append((x_to_dev(X), Wp, gd, N))
            cases.append((X, c, g))
        singles = [bl.bl_forward(Xd, Wp, gd, N, bits) for (Xd, Wp, gd, N) in probs]
        outs = bl.bl_forward_grouped(probs, bits)
        torch.cuda.synchronize()
        for (X, c, g), a, b in zip(cases, outs, singles):
            assert torch.equal(a, b)
            assert bf16_ulp_distance(bf16_dev_to_bits(a), oracle_bf16(X, c, g, bits)).max() <= BF16_ULP_TOL


def test_prepared_grouped_call_matches_and_sees_new_inputs():
    # the prepared form issues the same C call: equal outputs, and new input
    # contents (same buffers) are picked up by the next call
    cases = [(1, 2560, 700), (1, 2560, 33), (1, 6912, 130)]
    probs, Xs = [], []
    for j, (M, K, N) in enumerate(cases):
        X, W = random_case(M, K, N, seed=1300 + j)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        Xd = x_to_dev(X)
        probs.append((Xd, Wp, gd, N))
        Xs.append(Xd)
    call = bl.PreparedGrouped(probs)
    a = [y.clone() for y in call()]
    b = bl.bl_forward_grouped(probs)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    for j, Xd in enumerate(Xs):
        X2, _ = random_case(1, Xd.shape[1], 8, seed=1400 + j)
        Xd.copy_(x_to_dev(X2))
    c = [y.clone() for y in call()]
    d = bl.bl_forward_grouped(probs)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(c, d))
    assert not all(torch.equal(x, y) for x, y in zip(a, c))


@pytest.mark.parametrize("M", [1, 3, 130])
def test_grouped_host_buffers_match_device_path(M):
    # host-resident X and Y through bl_forward_grouped_host: one staged copy
    # for the shared input, the same kernels, outputs copied back
    shapes = [(2560, 700), (2560, 264), (6912, 130)]
    Xs, probs_d, probs_h, outs_h = {}, [], [], []
    for j, (K, N) in enumerate(shapes):
        X, W = random_case(M, K, N, seed=1500 + j)
        key = K
        if key not in Xs:
            Xs[key] = X
        Xh = torch.from_numpy(Xs[key].view(np.int16)).view(torch.bfloat16).pin_memory()
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs_d.append((x_to_dev(Xs[key]), Wp, gd, N))
        probs_h.append((Xh, Wp, gd, N))
        outs_h.append(torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory())
    # the two K = 2560 problems read one host tensor
    probs_h[1] = (probs_h[0][0],) + probs_h[1][1:]
    ref = bl.bl_forward_grouped(probs_d)
    call = bl.PreparedGroupedHost(probs_h, outs_h)
    for _ in range(2):
        call()
        torch.cuda.synchronize()
        for a, b in zip(outs_h, ref):
            assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))
    outs2 = [torch.empty_like(o).pin_memory() for o in outs_h]
    bl.bl_forward_grouped_host(probs_h, outs2)
    assert all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(outs2, outs_h))
    # inputs and outputs as adjacent views of one pinned buffer each: one
    # copy in and one copy out (the staged tensors keep their offsets)
    xin = torch.empty(M * (2560 + 6912), dtype=torch.bfloat16).pin_memory()
    xa, xb = xin[:M * 2560].view(M, 2560), xin[M * 2560:].view(M, 6912)
    xa.copy_(probs_h[0][0])
    xb.copy_(probs_h[2][0])
    yout = torch.full((M * (700 + 264 + 130),), float("nan"), dtype=torch.bfloat16).pin_memory()
    ys = [yout[:M * 700].view(M, 700), yout[M * 700:M * 964].view(M, 264), yout[M * 964:].view(M, 130)]
    adj = [(xa, probs_h[0][1], probs_h[0][2], 700), (xa, probs_h[1][1], probs_h[1][2], 264),
           (xb, probs_h[2][1], probs_h[2][2], 130)]
    a256 = lambda n: (n + 255) // 256 * 256   # noqa: E731 -- each run starts 256-byte aligned
    assert bl.bl_forward_grouped_host_staging_bytes(adj, ys) == a256(M * 9472 * 2) + a256(M * 1094 * 2)
    bl.PreparedGroupedHost(adj, ys)()
    torch.cuda.synchronize()
    for a, b in zip(ys, ref):
        assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))


@pytest.mark.parametrize("M", [1, 130])
def test_grouped_host_graph_replays_current_inputs(M):
    # the step recorded as a CUDA graph: each replay copies the host inputs'
    # current contents in and gives the outputs of a fresh device-path call
    shapes = [(2560, 700), (2560, 264), (6912, 130)]
    ws = []
    for j, (K, N) in enumerate(shapes):
        _, W = random_case(1, K, N, seed=1700 + j)
        ws.append(bl.bl_quantize_weights(torch.from_numpy(W).cuda()))
    xa = torch.empty((M, 2560), dtype=torch.bfloat16).pin_memory()
    xb = torch.empty((M, 6912), dtype=torch.bfloat16).pin_memory()
    xs = [xa, xa, xb]
    outs = [torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory() for _, N in shapes]
    probs_h = [(x, Wp, gd, N) for x, (Wp, gd), (_, N) in zip(xs, ws, shapes)]
    for trial in range(3):
        xa.copy_(torch.from_numpy(random_case(M, 2560, 1, seed=1800 + trial)[0].view(np.int16)).view(torch.bfloat16))
        xb.copy_(torch.from_numpy(random_case(M, 6912, 1, seed=1900 + trial)[0].view(np.int16)).view(torch.bfloat16))
        if trial == 0:
            call = bl.PreparedGroupedHost(probs_h, outs, graph=True)   # records (and runs) the step
        else:
            call()
        torch.cuda.synchronize()
        ref = bl.bl_forward_grouped([(x.cuda(), Wp, gd, N) for x, (Wp, gd), (_, N) in zip(xs, ws, shapes)])
        for a, b in zip(outs, ref):
            assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16)), trial
    del call


def test_grouped_mixed_shapes_fall_back_to_sequential():
    cases = [(1, 256, 300), (3, 512, 129), (1, 4096, 64), (2, 192, 100), (0, 64, 8)]
    probs, singles = [], []
    for j, (M, K, N) in enumerate(cases):
        X, W = random_case(M, K, N, seed=100 + j)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        Xd = x_to_dev(X) if M > 0 else torch.zeros((0, K), dtype=torch.bfloat16, device="cuda")
        probs.append((Xd, Wp, gd, N))
        singles.append(bl.bl_forward(Xd, Wp, gd, N))
    outs = bl.bl_forward_grouped(probs)
    torch.cuda.synchronize()
    for a, b in zip(outs, singles):
        assert torch.equal(a, b)
    # all-decode group of different K (one launch)
    probs2 = [probs[0], probs[2]]
    outs2 = bl.bl_forward_grouped(probs2)
    assert torch.equal(outs2[0], singles[0]) and torch.equal(outs2[1], singles[2])
    # several one-token problems of one kernel variant with ragged row counts
    probs3, singles3 = [], []
    for j, (K, N) in enumerate([(2560, 6912), (2560, 33), (2048, 1000), (2560, 1)]):
        X, W = random_case(1, K, N, seed=300 + j)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs3.append((x_to_dev(X), Wp, gd, N))
        singles3.append(bl.bl_forward(probs3[-1][0], Wp, gd, N))
    outs3 = bl.bl_forward_grouped(probs3)
    for a, b in zip(outs3, singles3):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M,K,N1,N2", [(3, 512, 300, 129), (64, 1024, 520, 256), (65, 512, 130, 1000),
                                        (130, 2560, 1000, 264), (257, 640, 6912, 8), (300, 256, 7, 2049)])
def test_grouped_shared_input_pair(M, K, N1, N2):
    # two projections of one X (the up and gate shape) share the activation
    # quantisation and, past 64 tokens, one tensor-core launch over both
    # weight tensors; a third problem with its own X sits between them; ragged
    # M and N, N not a multiple of 8 (plain epilogue stores) and of 256 (a
    # partial last tile in either weight tensor)
    X, W1 = random_case(M, K, N1, seed=700 + M)
    _, W2 = random_case(M, K, N2, seed=800 + M)
    X3, W3 = random_case(M, K, 96, seed=900 + M)
    Xd = x_to_dev(X)
    probs, cases = [], []
    for Xh, Xt, W in ((X, Xd, W1), (X3, x_to_dev(X3), W3), (X, Xd, W2)):
        g = o.absmean_scale(W)
        c = o.ternary_codes(W, g)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs.append((Xt, Wp, gd, W.shape[0]))
        cases.append((Xh, c, g))
    for bits in (8, 4):
        singles = [bl.bl_forward(Xt, Wp, gd, N, bits) for (Xt, Wp, gd, N) in probs]
        outs = bl.bl_forward_grouped(probs, bits)
        outs = bl.bl_forward_grouped(probs, bits, outs=outs)   # twice in a row, outputs reused
        torch.cuda.synchronize()
        for (Xh, c, g), a, b in zip(cases, outs, singles):
            assert torch.equal(a, b)
            assert bf16_ulp_distance(bf16_dev_to_bits(a), oracle_bf16(Xh, c, g, bits)).max() <= BF16_ULP_TOL


def test_grouped_shared_input_pair_prefill_full_size():
    # the 2B prefill up and gate projections (4096 tokens, K = 2560, N = 6912
    # each) in one tensor-core launch: equal to two single calls everywhere,
    # and to the oracle on sampled rows
    w = WORKLOADS["prefill_2b"]
    X, _ = layer_inputs(w, 0)
    Xd = x_to_dev(X)
    probs, cases = [], []
    W_up, _, _, _ = oracle_weights(("prefill_2b", 0))
    for W in (W_up, make_weight(W_up.shape[0], W_up.shape[1], 0.02, 4321)):
        g = o.absmean_scale(W)
        c = o.ternary_codes(W, g)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs.append((Xd, Wp, gd, W.shape[0]))
        cases.append((c, g))
    singles = [bl.bl_forward(Xd, Wp, gd, N) for (_, Wp, gd, N) in probs]
    outs = bl.bl_forward_grouped(probs)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(7).choice(X.shape[0], 24, replace=False))
    for (c, g), a, b in zip(cases, outs, singles):
        assert torch.equal(a, b)
        ref = oracle_bf16(X[rows], c, g)
        assert bf16_ulp_distance(bf16_dev_to_bits(a[torch.from_numpy(rows).cuda()]), ref).max() <= BF16_ULP_TOL


# ---------------------------------------------------------------------------
# squared-ReLU feed-forward input ("BitNet 2B4T Guide: Scaling Native 1.58-Bit
# LLMs", section "2. Squared ReLU Activation")
# ---------------------------------------------------------------------------

def relu2_inputs(M, K, N, seed):
    G, W = random_case(M, K, N, seed=seed)
    U, _ = random_case(M, K, 8, seed=seed + 7)
    return G, U, W


@pytest.mark.parametrize("M,K", [(1, 64), (3, 192), (16, 2560), (5, 6912), (2, 8192)])
@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("bits", [8, 4])
def test_quant_act_relu2_bit_exact(M, K, gated, bits):
    G, U, _ = relu2_inputs(M, K, 8, seed=M * 31 + K)
    h = o.relu2_input(G, U if gated else None)
    q, s = o.act_quant_values(h, bits)
    qd, sd = bl.bl_quant_act_relu2(x_to_dev(G), x_to_dev(U) if gated else None, bits)
    assert np.array_equal(qd.cpu().numpy(), q)
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s.view(np.uint32))


RELU2_CASES = [(1, 2560, 700), (1, 6912, 2560), (1, 8192, 2100), (1, 8192, 8192), (1, 16384, 64),
               (2, 320, 130), (3, 256, 512), (17, 320, 130), (130, 256, 300), (16, 4096, 300)]


@pytest.mark.parametrize("M,K,N", RELU2_CASES)
@pytest.mark.parametrize("gated", [False, True])
def test_forward_relu2_parity(M, K, N, gated):
    # one token: the decode kernels (resident for small layers, streaming for
    # 8192 x 8192) form h in their prologue; otherwise the quantiser + GEMM
    G, U, W = relu2_inputs(M, K, N, seed=M * 1000 + K + N)
    ref = o.forward_relu2(G, U if gated else None, W)
    Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
    Yd = bl.bl_forward_relu2(x_to_dev(G), x_to_dev(U) if gated else None, Wp, gd, N)
    torch.cuda.synchronize()
    d = bf16_ulp_distance(bf16_dev_to_bits(Yd), ref["Y"])
    assert d.max() <= BF16_ULP_TOL, f"bf16 ulp distance {d.max()}"
    # the same arithmetic as the oracle: almost every output is bit-identical
    assert np.mean(d == 0) > 0.99


def test_forward_relu2_bits4_and_zero_rows():
    M, K, N = 4, 512, 96
    G, U, W = relu2_inputs(M, K, N, seed=77)
    G[1] = 0x8000          # -0.0 everywhere: relu^2 is all zero -> zero codes, Y = 0
    G[2] = 0xBF80          # -1.0 everywhere: also all zero
    for bits in (8, 4):
        ref = o.forward_relu2(G, U, W, bits)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        Yd = bf16_dev_to_bits(bl.bl_forward_relu2(x_to_dev(G), x_to_dev(U), Wp, gd, N, bits))
        assert bf16_ulp_distance(Yd, ref["Y"]).max() <= BF16_ULP_TOL
        assert np.all(Yd[1] == 0) and np.all(Yd[2] == 0)


# ---------------------------------------------------------------------------
# per-tensor activation scale and output bias (bl_forward_ex)
# ---------------------------------------------------------------------------

EX_CASES = [(1, 2560, 700), (1, 8192, 8192), (1, 16384, 64), (2, 320, 130), (3, 256, 512), (17, 320, 130),
            (130, 256, 300), (300, 1024, 700), (16, 4096, 300)]


@pytest.mark.parametrize("M,K,N", EX_CASES)
@pytest.mark.parametrize("per_tensor,with_bias", [(True, False), (False, True), (True, True)])
def test_forward_ex_parity(M, K, N, per_tensor, with_bias):
    X, W = random_case(M, K, N, seed=M * 7 + K + N)
    bias = (np.random.default_rng(N).standard_normal(N) * 0.5).astype(np.float32) if with_bias else None
    for bits in ((8, 4) if M in (3, 130) else (8,)):
        ref = o.forward_ex(X, W, bits, per_tensor=per_tensor, bias=bias)
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        Yd = bl.bl_forward_ex(x_to_dev(X), Wp, gd, N, bits, per_tensor=per_tensor,
                              bias=torch.from_numpy(bias).cuda() if bias is not None else None)
        torch.cuda.synchronize()
        d = bf16_ulp_distance(bf16_dev_to_bits(Yd), ref["Y"])
        assert d.max() <= BF16_ULP_TOL, f"bf16 ulp distance {d.max()}"
        assert np.mean(d == 0) > 0.99


# ---------------------------------------------------------------------------
# RMSNorm before the quantisation ("BitNet 2B4T Guide: Scaling Native 1.58-Bit
# LLMs", section "3. Sub-Layer Normalization (SubLN)")
# ---------------------------------------------------------------------------

def norm_weight_bits(K, seed):
    w = np.random.default_rng(seed).uniform(0.25, 2.0, size=K).astype(np.float32)
    return (w.view(np.uint32) >> 16).astype(np.uint16)   # truncation: any bf16 will do


def check_quant_rmsnorm(X, wb, eps, bits):
    nrm = o.rms_norm(X, wb, eps)
    q, s = o.act_quant(nrm["xn"], bits)
    qd, sd, msd = bl.bl_quant_act_rmsnorm(x_to_dev(X), bits, x_to_dev(wb) if wb is not None else None, eps)
    assert np.array_equal(msd.cpu().numpy().view(np.uint32), nrm["ms"].view(np.uint32))
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(qd.cpu().numpy(), q)


@pytest.mark.parametrize("M,K", [(1, 64), (3, 192), (16, 2560), (5, 6912), (2, 8192), (2, 20480), (1, 65536)])
@pytest.mark.parametrize("with_weight", [False, True])
@pytest.mark.parametrize("bits", [8, 4])
def test_quant_act_rmsnorm_bit_exact(M, K, with_weight, bits):
    X, _ = random_case(M, K, 8, seed=M * 17 + K)
    check_quant_rmsnorm(X, norm_weight_bits(K, K) if with_weight else None, 1e-5, bits)


def test_quant_act_rmsnorm_hard_sums():
    rng = np.random.default_rng(2024)
    K = 2560
    rows = []
    rows.append(rng.integers(0, 0x7F80, K).astype(np.uint16))              # every exponent: many far terms
    x = rng.standard_normal(K).astype(np.float32)
    x[rng.integers(0, K, K // 3)] *= 1e-25                                 # a third far below the rest
    rows.append((x.view(np.uint32) >> 16).astype(np.uint16))
    rows.append(rng.integers(0x2000, 0x5F00, K).astype(np.uint16))         # 2^-63 .. 2^63: far terms, finite ms
    rows.append(rng.integers(0x1A00, 0x2000, K).astype(np.uint16))         # 2^-75 .. 2^-63: subnormal ms
    rows.append(rng.integers(0, 0x100, K).astype(np.uint16))               # bf16 subnormals: ms rounds to 0
    big = np.zeros(K, np.uint16)
    big[[3, 900]] = 0x7149                                                 # ~1e30: ms overflows to inf
    rows.append(big)
    rows.append(np.zeros(K, np.uint16))                                    # zero row
    X = np.stack(rows) | (rng.integers(0, 2, (len(rows), K)).astype(np.uint16) << 15)
    for eps in (1e-5, 1e-30):
        check_quant_rmsnorm(X, None, eps, 8)
    # an exact midpoint of two fp32 values (ties to even), and just above it
    v = np.zeros((2, 128), np.float32)
    v[:, :64] = 1.0
    v[:, 64] = 2.0 ** -9
    v[1, 65] = 2.0 ** -60
    Xm = (v.view(np.uint32) >> 16).astype(np.uint16)
    check_quant_rmsnorm(Xm, None, 2.0 ** -40, 8)
    _, _, msd = bl.bl_quant_act_rmsnorm(x_to_dev(Xm), 8, None, 2.0 ** -40)
    assert msd.cpu().numpy().tolist() == [0.5, 0.5 + 2.0 ** -24]


RMS_CASES = [(1, 2560, 6912), (1, 6912, 2560), (1, 8192, 2100), (1, 8192, 8192), (1, 16384, 64),
             (2, 320, 130), (17, 320, 130), (130, 256, 300), (16, 4096, 300)]


@pytest.mark.parametrize("M,K,N", RMS_CASES)
@pytest.mark.parametrize("with_weight", [False, True])
def test_forward_rmsnorm_parity(M, K, N, with_weight):
    # one token with a layer that fits the resident decode kernel: RMSNorm in
    # its prologue; otherwise the normalising quantiser + the tensor-core GEMM
    X, W = random_case(M, K, N, seed=M * 3 + K + N)
    wb = norm_weight_bits(K, N) if with_weight else None
    ref = o.forward_rmsnorm(X, W, wb, 1e-5)
    Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
    Yd = bf16_dev_to_bits(bl.bl_forward_rmsnorm(x_to_dev(X), Wp, gd, N, norm_weight=x_to_dev(wb) if wb is not None
                                                else None, eps=1e-5))
    d = bf16_ulp_distance(Yd, ref["Y"])
    assert d.max() <= BF16_ULP_TOL, f"bf16 ulp distance {d.max()}"
    assert np.mean(d == 0) > 0.99
    # and bit-identical to bl_forward on the oracle's normalised bf16 input
    Y2 = bf16_dev_to_bits(bl.bl_forward(x_to_dev(ref["xn"]), Wp, gd, N))
    assert np.array_equal(Yd, Y2)


def test_forward_rmsnorm_bits4_zero_rows_and_back_to_back():
    M, K, N = 1, 2560, 700
    X, W = random_case(3, K, N, seed=99)
    X[1] = 0
    Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
    ws = torch.empty(bl.bl_forward_rmsnorm_workspace_bytes(M, K, N, 4), dtype=torch.uint8, device="cuda")
    outs = []
    for m in range(3):   # three decode launches back to back on one stream
        outs.append(bl.bl_forward_rmsnorm(x_to_dev(X[m:m + 1]), Wp, gd, N, bits=4, workspace=ws))
    torch.cuda.synchronize()
    for m in range(3):
        ref = o.forward_rmsnorm(X[m:m + 1], W, None, 1e-5, bits=4)
        d = bf16_ulp_distance(bf16_dev_to_bits(outs[m]), ref["Y"])
        assert d.max() <= BF16_ULP_TOL
    assert np.all(bf16_dev_to_bits(outs[1]) == 0)


# ---------------------------------------------------------------------------
# LayerNorm before the quantisation ("BitNet b1.58: The 1-Bit Ternary LLM
# Architecture Guide", BitLinear code listing, forward step 1)
# ---------------------------------------------------------------------------

def bf16_bits_of(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def check_quant_layernorm(X, eps, bits):
    nrm = o.layer_norm(X, eps)
    q, s = o.act_quant(nrm["xn"], bits)
    qd, sd, mud, vard = bl.bl_quant_act_layernorm(x_to_dev(X), bits, eps)
    assert np.array_equal(mud.cpu().numpy().view(np.uint32), nrm["mean"].view(np.uint32))
    assert np.array_equal(vard.cpu().numpy().view(np.uint32), nrm["var"].view(np.uint32))
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(qd.cpu().numpy(), q)


@pytest.mark.parametrize("M,K", [(1, 64), (3, 192), (16, 2560), (5, 6912), (2, 8192), (2, 20480), (1, 65536)])
@pytest.mark.parametrize("bits", [8, 4])
def test_quant_act_layernorm_bit_exact(M, K, bits):
    # per-row offsets make the mean matter next to the spread
    X, _ = random_case(M, K, 8, seed=M * 19 + K)
    off = np.random.default_rng(K + M).uniform(-6, 6, size=(M, 1))
    X = bf16_bits_of(o.bf16_bits_to_f32(X) + off)
    check_quant_layernorm(X, 1e-5, bits)


def test_quant_act_layernorm_hard_sums():
    rng = np.random.default_rng(2025)
    K = 2560
    rows = []
    rows.append(rng.integers(0, 0x7F80, K).astype(np.uint16))              # every exponent: far terms
    x = rng.standard_normal(K).astype(np.float32) + 3.0
    x[rng.integers(0, K, K // 3)] *= 1e-25                                 # a third far below the rest
    rows.append((x.view(np.uint32) >> 16).astype(np.uint16))
    rows.append(rng.integers(0x2000, 0x5F00, K).astype(np.uint16))         # 2^-63 .. 2^63
    rows.append(rng.integers(0x1A00, 0x2000, K).astype(np.uint16))         # 2^-75 .. 2^-63: subnormal var
    rows.append(rng.integers(0, 0x100, K).astype(np.uint16))               # bf16 subnormals: subnormal mean
    big = np.zeros(K, np.uint16)
    big[[3, 900]] = 0x7149                                                 # ~1e30: var overflows to inf
    rows.append(big)
    rows.append(np.zeros(K, np.uint16))                                    # zero row
    rows.append(np.full(K, 0x4060, np.uint16))                             # constant 3.5: var 0
    near = np.full(K, 0x4060, np.uint16)
    near[7] = 0x4061                                                       # one value one step away
    rows.append(near)
    X = np.stack(rows)
    X[:5] |= (rng.integers(0, 2, (5, K)).astype(np.uint16) << 15)
    for eps in (1e-5, 1e-30):
        check_quant_layernorm(X, eps, 8)
    # exact fp32 midpoints of the mean (ties to even), and just above one
    v = np.zeros((3, 128), np.float32)
    v[:, 0] = v[:, 1] = 64.0
    v[:2, 2] = 2.0 ** -17                                                  # sum 128 + 2^-17, K = 128:
    #                                                                        mean 1 + 2^-24, a tie -> 1
    v[1, 3] = 2.0 ** -100                                                  # just above -> 1 + 2^-23
    v[2, 2], v[2, 3] = 2.0 ** -16, 2.0 ** -17                              # mean 1 + 3 2^-24: tie -> 1 + 2^-22
    Xm = (v.view(np.uint32) >> 16).astype(np.uint16)
    check_quant_layernorm(Xm, 2.0 ** -40, 8)
    _, _, mud, _ = bl.bl_quant_act_layernorm(x_to_dev(Xm), 8, 2.0 ** -40)
    assert mud.cpu().numpy().tolist() == [1.0, 1.0 + 2.0 ** -23, 1.0 + 2.0 ** -22]


@pytest.mark.parametrize("M,K,N", RMS_CASES)
def test_forward_layernorm_parity(M, K, N):
    # one token with a layer that fits the resident decode kernel: LayerNorm
    # in its prologue; otherwise the normalising quantiser + the tensor-core GEMM
    X, W = random_case(M, K, N, seed=M * 5 + K + N)
    X = bf16_bits_of(o.bf16_bits_to_f32(X) + np.float32(1.5))
    ref = o.forward_layernorm(X, W, 1e-5)
    Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
    Yd = bf16_dev_to_bits(bl.bl_forward_layernorm(x_to_dev(X), Wp, gd, N, eps=1e-5))
    d = bf16_ulp_distance(Yd, ref["Y"])
    assert d.max() <= BF16_ULP_TOL, f"bf16 ulp distance {d.max()}"
    assert np.mean(d == 0) > 0.99
    Y2 = bf16_dev_to_bits(bl.bl_forward(x_to_dev(ref["xn"]), Wp, gd, N))
    assert np.array_equal(Yd, Y2)


@pytest.mark.parametrize("norm", ["rms", "layer"])
def test_norm_grouped_decode_one_launch(norm):
    # the 2B decode step with a normalisation ahead of every projection, one
    # launch: up and gate read the same X, down its own; RMSNorm weights
    # differ per problem; bits 8 and 4
    w = WORKLOADS["decode_2b"]
    probs, cases, nws = [], [], []
    xs = {}
    for i, L in enumerate(w.layers):
        X, _ = layer_inputs(w, i)
        key = L.x_layer if L.x_layer >= 0 else i
        if key not in xs:
            xs[key] = (X, x_to_dev(X))
        Xh, Xd = xs[key]
        W, g, c, _ = oracle_weights(("decode_2b", i))
        Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
        probs.append((Xd, Wp, gd, W.shape[0]))
        wb = norm_weight_bits(L.K, 31 + i) if norm == "rms" else None
        nws.append(x_to_dev(wb) if wb is not None else None)
        cases.append((Xh, W, wb))
    kind = bl.BL_NORM_RMS if norm == "rms" else bl.BL_NORM_LAYER
    for bits in (8, 4):
        if norm == "rms":
            singles = [bl.bl_forward_rmsnorm(Xd, Wp, gd, N, bits, norm_weight=nw) for (Xd, Wp, gd, N), nw in
                       zip(probs, nws)]
        else:
            singles = [bl.bl_forward_layernorm(Xd, Wp, gd, N, bits) for (Xd, Wp, gd, N) in probs]
        outs = bl.bl_forward_norm_grouped(probs, kind, nws if norm == "rms" else None, bits=bits)
        outs = bl.bl_forward_norm_grouped(probs, kind, nws if norm == "rms" else None, bits=bits, outs=outs)
        torch.cuda.synchronize()
        for (Xh, W, wb), a, b in zip(cases, outs, singles):
            assert torch.equal(a, b)
            ref = o.forward_rmsnorm(Xh, W, wb, 1e-5, bits) if norm == "rms" else o.forward_layernorm(Xh, W, 1e-5, bits)
            assert bf16_ulp_distance(bf16_dev_to_bits(a), ref["Y"]).max() <= BF16_ULP_TOL


def test_norm_grouped_sequential_shapes():
    # problems that do not fit one decode launch (several tokens, long rows)
    cases = [(3, 256, 300), (1, 16384, 64), (1, 2560, 700), (0, 64, 8), (130, 512, 264)]
    for kind in (bl.BL_NORM_RMS, bl.BL_NORM_LAYER):
        probs, singles = [], []
        for j, (M, K, N) in enumerate(cases):
            X, W = random_case(M, K, N, seed=600 + j)
            Wp, gd = bl.bl_quantize_weights(torch.from_numpy(W).cuda())
            Xd = x_to_dev(X) if M > 0 else torch.zeros((0, K), dtype=torch.bfloat16, device="cuda")
            probs.append((Xd, Wp, gd, N))
            singles.append(bl.bl_forward_rmsnorm(Xd, Wp, gd, N) if kind == bl.BL_NORM_RMS
                           else bl.bl_forward_layernorm(Xd, Wp, gd, N))
        outs = bl.bl_forward_norm_grouped(probs, kind)
        torch.cuda.synchronize()
        for a, b in zip(outs, singles):
            assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# packed 4-bit activations ("BitNet a4.8 Guide: 4-Bit Activation 1-Bit LLMs",
# section "Step 4: Verification and Benchmarking Test Harness")
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,K", [(1, 64), (3, 4096), (7, 8192), (2, 65536)])
def test_quant_act_packed4_bit_exact(M, K):
    X, _ = random_case(M, K, 8, seed=700 + M + K, x_kind="relu2")
    q, s = o.act_quant(X, 4)
    p4, sd = bl.bl_quant_act_packed4(x_to_dev(X))
    assert np.array_equal(p4.cpu().numpy(), o.pack_int4(q))
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s.view(np.uint32))


def test_quant_act_packed4_a48_full_size():
    w = WORKLOADS["a48"]
    X, _ = layer_inputs(w, 0)
    q, s = o.act_quant(X, 4)
    p4, sd = bl.bl_quant_act_packed4(x_to_dev(X))
    assert np.array_equal(p4.cpu().numpy(), o.pack_int4(q))
    # the same codes as the one-byte-a-code quantiser
    qd, _ = bl.bl_quant_act(x_to_dev(X), 4)
    assert np.array_equal(o.unpack_int4(p4.cpu().numpy(), X.shape[1]), qd.cpu().numpy())
