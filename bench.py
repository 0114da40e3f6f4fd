"""BitLinear forward benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Headline workload: the 2B-class decode layer set (batch 1; up and gate
2560 -> 6912, down 6912 -> 2560).  A step is one pass of the forward hot path
(per-token quantisation, ternary GEMV, rescale to bf16) over all three layers.
Weights are quantised once before timing (the offline part of the method, timed
separately).  Metric: HBM GB/s of algorithmic bytes
(packed weights + bf16 activations in + bf16 out + scales).  Secondary lines
report tensor-core TOPS on the prefill workloads.

Timing: CUDA graphs of back-to-back steps, CUDA events on the launching stream,
barrier + synchronize on both sides of exactly K steps, max over ranks.  Each
step uses one of several rotated copies of the weights so the weight stream is
larger than the 126 MB L2.  With --gpus N > 1 (torchrun), every rank runs an
independent replica (the decode path has no exchange step), and the value is
the work of all ranks over the slowest rank's time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BitLinear TOPS (prefill) and HBM GB/s (decode) vs roofline, 1×B200"
INT8_NOMINAL_RATIO = 2.0   # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
DELAY_CYCLES = 400_000     # ~200 us at the 1965 MHz maximum SM clock


# ---------------------------------------------------------------------------
# shared helpers
# ---------------------------------------------------------------------------

def algorithmic_bytes(M, K, N):
    """Packed weights + bf16 X + bf16 Y + fp32 scales and gamma."""
    return N * K // 4 + 2 * M * K + 2 * M * N + 4 * M + 4


def algorithmic_ops(M, K, N):
    return 2 * M * N * K


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def ncu_traffic(kernel_key):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the kernel's current source (hash of the source files the line lists);
    otherwise None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    src = os.path.join(ROOT, "bitlinear_bl_forward_b200", "csrc")
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(t.split("=", 1) for t in line.split())
        if kv.get("key") != kernel_key or "files" not in kv:
            continue
        h = hashlib.sha256()
        for fn in kv["files"].split(","):
            fp = os.path.join(src, fn)
            if not os.path.exists(fp):    # the kernel's sources changed since the capture
                return None
            h.update(open(fp, "rb").read())
        if kv.get("src_sha") == h.hexdigest()[:16]:
            return float(kv["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        time.sleep(0.15)
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            p = [t.strip() for t in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), float(p[3]), p[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        busy = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(busy),
                "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# the oracle arm (CPU): the CPU baseline and --impl reference
# ---------------------------------------------------------------------------

def oracle_step_fn(workload_name, row_fraction=1.0):
    """Return (fn, bytes_per_call, ops_per_call, description): fn() runs the oracle's forward
    scope (activation quantisation, integer matmul, rescale, bf16 rounding)
    over every layer of the workload, restricted to the first
    ceil(row_fraction * N) output features of each layer."""
    from bitlinear_bl_forward_b200.inputs import WORKLOADS, layer_inputs
    from oracle import bitlinear_oracle as o
    w = WORKLOADS[workload_name]
    layers = []
    nbytes = 0
    ops = 0
    for i, L in enumerate(w.layers):
        X, W = layer_inputs(w, i)
        n = max(1, int(math.ceil(row_fraction * L.N)))
        W = W[:n]
        g = o.absmean_scale(W)
        c = o.ternary_codes(W, g)
        layers.append((X, g, c))
        # an input shared with an earlier layer (same hidden state) is counted once, as on the GPU arm
        nbytes += algorithmic_bytes(w.M, L.K, n) - (2 * w.M * L.K if L.x_layer >= 0 else 0)
        ops += algorithmic_ops(w.M, L.K, n)

    def fn():
        for X, g, c in layers:
            q, s = o.act_quant(X, w.bits)
            acc = o.matmul_i32(q, c)
            _, y32 = o.rescale(acc, g, s)
            o.round_to_bf16_bits(y32)

    desc = f"{workload_name}, first {row_fraction:.4g} of each layer's output rows"
    return fn, nbytes, ops, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _time_oracle(fn, budget_s):
    fn()   # warm
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(workload_name, budget_s=8.0):
    """The oracle's forward scope on the host cores, twice: with the BLAS pool
    (the oracle's float64 matmul) limited to one thread, and with all of it.
    The oracle's quantisation and rescale are single-threaded numpy in both."""
    from threadpoolctl import threadpool_limits
    fn, nbytes, _ops, desc = oracle_step_fn(workload_name)
    with threadpool_limits(limits=1, user_api="blas"):
        n1, dt1 = _time_oracle(fn, budget_s)
    n, dt = _time_oracle(fn, budget_s)
    cores = blas_threads()
    return {"value": nbytes * n / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} full steps of {desc} in {dt:.1f} s with {cores} BLAS threads (weight quantisation "
                      f"excluded; the oracle's quantiser and rescale are single-threaded numpy)",
            "single_thread": {"value": nbytes * n1 / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"{n1} full steps in {dt1:.1f} s, BLAS limited to 1 thread"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload
    K, W = args.steps, args.warmup
    # calibrate one full step, then size each step so the run stays within ~2 minutes
    fn, nbytes, ops, _ = oracle_step_fn(name)
    t0 = time.perf_counter()
    fn()
    t_full = time.perf_counter() - t0
    frac = min(1.0, 120.0 / max(1e-9, (K + W) * t_full))
    if frac < 1.0:
        fn, nbytes, ops, _ = oracle_step_fn(name, frac)
    for _ in range(W):
        fn()
    t0 = time.perf_counter()
    for _ in range(K):
        fn()
    dt = time.perf_counter() - t0
    from bitlinear_bl_forward_b200.inputs import WORKLOADS
    w = WORKLOADS[name]
    decode = w.M <= 2
    unit = "GB/s" if decode else "TOPS"
    value = (nbytes * K / dt / 1e9) if decode else (ops * K / dt / 1e12)
    cores = blas_threads()
    groups = [list(gr) for gr in w.groups] or [[i] for i in range(len(w.layers))]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": K,
        "warmup": W, "ms_per_step": dt / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic (seeded; the oracle on the host cores)",
        "config": {"workload": name, "M": w.M, "layers": [[L.name, L.K, L.N] for L in w.layers], "bits": w.bits,
                   "calls_per_step": [[w.layers[j].name for j in gr] for gr in groups],
                   "parallelism": "host cores (rank 0 only)"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {name}, fraction {frac:.4g} of each layer's output rows"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------

class GpuWorkload:
    """Device buffers for one workload: R rotated copies of the packed weights
    of every layer, one bf16 input and output per layer, workspace."""

    def __init__(self, name, rotations, seed=0, device="cuda", fmt="2bit"):
        import torch
        from bitlinear_bl_forward_b200 import bl
        from bitlinear_bl_forward_b200.inputs import WORKLOADS, make_activation
        self.w = WORKLOADS[name]
        self.name = name
        self.fmt = fmt
        self.layers = []
        g = torch.Generator(device=device).manual_seed(seed)
        for i, L in enumerate(self.w.layers):
            Wf = torch.randn(L.N, L.K, generator=g, device=device, dtype=torch.float32) * self.w.w_std
            Wp, gamma = (bl.bl_quantize_weights_b3 if fmt == "b3" else bl.bl_quantize_weights)(Wf)
            del Wf
            copies = [(Wp, gamma)] + [(Wp.clone(), gamma.clone()) for _ in range(rotations - 1)]
            if L.x_layer >= 0:          # reads the same hidden state as an earlier layer
                src = self.layers[L.x_layer]
                xb, X, own_x = src["xb"], src["X"], False
            else:
                xb = make_activation(self.w.M, L.K, self.w.x_kind, seed + 1 + 10 * i, self.w.outliers_for(L.K),
                                     self.w.outlier_mult)
                X, own_x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(device), True
            Y = torch.empty((self.w.M, L.N), dtype=torch.bfloat16, device=device)
            ws_n = bl.bl_forward_workspace_bytes(self.w.M, L.K, L.N, self.w.bits)
            ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=device)
            self.layers.append(dict(L=L, copies=copies, X=X, Y=Y, ws=ws, xb=xb, own_x=own_x))
        self.rotations = rotations
        self.prepared = {}
        # layers run together in one grouped call (e.g. up and gate of a feed-forward block)
        self.groups = [list(gr) for gr in self.w.groups] or [[i] for i in range(len(self.layers))]
        self.group_ws = []
        for gr in self.groups:
            if len(gr) > 1:
                probs = [(self.layers[j]["X"], *self.layers[j]["copies"][0], self.layers[j]["L"].N) for j in gr]
                n = bl.bl_forward_grouped_workspace_bytes(probs, self.w.bits)
                self.group_ws.append(torch.empty(max(n, 16), dtype=torch.uint8, device=device))
            else:
                self.group_ws.append(None)
        # activations shared by several layers are read (and counted) once
        self.bytes_per_step = sum(algorithmic_bytes(self.w.M, d["L"].K, d["L"].N)
                                  - (0 if d["own_x"] else 2 * self.w.M * d["L"].K) for d in self.layers)
        if fmt == "b3":   # the stored weight bytes are the base-3 rows
            self.bytes_per_step += sum(bl.bl_packed_weight_bytes_b3(d["L"].N, d["L"].K) - d["L"].N * d["L"].K // 4
                                       for d in self.layers)
        self.ops_per_step = sum(algorithmic_ops(self.w.M, d["L"].K, d["L"].N) for d in self.layers)
        # decode: one launch per call (a grouped call of decode problems is one launch);
        # otherwise activation quantisation + GEMM per layer
        self.launches_per_step = len(self.groups) if self.w.M <= 2 else 2 * len(self.layers)

    def run_group(self, gi, r):
        from bitlinear_bl_forward_b200 import bl
        gr = self.groups[gi]
        if len(gr) == 1:
            d = self.layers[gr[0]]
            Wp, gamma = d["copies"][r]
            if self.fmt == "b3":
                bl.bl_forward_b3(d["X"], Wp, gamma, d["L"].N, self.w.bits, out=d["Y"])
            else:
                bl.bl_forward(d["X"], Wp, gamma, d["L"].N, self.w.bits, out=d["Y"], workspace=d["ws"])
        else:
            # the grouped call prepared once per rotation (argument packing
            # outside the step); rebuilt when a layer's buffers are replaced
            ds = [self.layers[j] for j in gr]
            key = (gi, r, tuple(d["X"].data_ptr() for d in ds), tuple(d["Y"].data_ptr() for d in ds))
            call = self.prepared.get(key)
            if call is None:
                call = bl.PreparedGrouped([(d["X"], *d["copies"][r], d["L"].N) for d in ds], self.w.bits,
                                          outs=[d["Y"] for d in ds], workspace=self.group_ws[gi])
                self.prepared[key] = call
            call()

    def step(self, i):
        r = i % self.rotations
        for gi in range(len(self.groups)):
            self.run_group(gi, r)

class FfnWorkload(GpuWorkload):
    """The 2B decode feed-forward block as a chain: up and gate in one grouped
    launch, then the down projection on max(0, gate)^2 * up formed and
    quantised in the down kernel's prologue (its input is the previous
    launch's output)."""

    def __init__(self, rotations, seed=0, device="cuda"):
        super().__init__("decode_2b", rotations, seed, device)
        up, gate, down = self.layers
        self.groups = [[0, 1], [2]]
        self.bytes_per_step = (algorithmic_bytes(1, up["L"].K, up["L"].N)
                               + algorithmic_bytes(1, gate["L"].K, gate["L"].N) - 2 * gate["L"].K
                               + algorithmic_bytes(1, down["L"].K, down["L"].N) + 2 * down["L"].K)
        self.launches_per_step = 2

    def step(self, i):
        from bitlinear_bl_forward_b200 import bl
        r = i % self.rotations
        self.run_group(0, r)
        up, gate, down = self.layers
        Wp, gamma = down["copies"][r]
        bl.bl_forward_relu2(gate["Y"], up["Y"], Wp, gamma, down["L"].N, self.w.bits, out=down["Y"],
                            workspace=down["ws"])


class NormWorkload(GpuWorkload):
    """Every layer of a workload with a normalisation ahead of its quantiser:
    RMSNorm with a bf16 weight [K] per layer, or LayerNorm without parameters.
    One-token steps issue one bl_forward_norm_grouped call over all layers
    (one launch); otherwise one bl_forward_rmsnorm / bl_forward_layernorm call
    per layer (normalising quantiser + GEMM)."""

    def __init__(self, name, rotations, norm, seed=0, device="cuda"):
        import torch
        from bitlinear_bl_forward_b200 import bl
        super().__init__(name, rotations, seed, device)
        self.norm = norm
        g = torch.Generator(device=device).manual_seed(seed + 99)
        for d in self.layers:
            L = d["L"]
            d["nw"] = ((torch.rand(L.K, generator=g, device=device) + 0.5).to(torch.bfloat16)
                       if norm == bl.BL_NORM_RMS else None)
            n = bl.bl_forward_rmsnorm_workspace_bytes(self.w.M, L.K, L.N, self.w.bits)
            d["ws"] = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
        self.one_call = self.w.M == 1
        if self.one_call:
            probs = [(d["X"], *d["copies"][0], d["L"].N) for d in self.layers]
            n = bl.bl_forward_norm_grouped_workspace_bytes(probs, self.w.bits)
            self.gws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
            self.groups = [list(range(len(self.layers)))]
        else:
            self.groups = [[i] for i in range(len(self.layers))]
        # every layer normalises its own copy of the input: a shared X is read per layer
        self.bytes_per_step = sum(algorithmic_bytes(self.w.M, d["L"].K, d["L"].N)
                                  + (2 * d["L"].K if norm == bl.BL_NORM_RMS else 0) for d in self.layers)
        self.launches_per_step = 1 if self.one_call else 2 * len(self.layers)

    def step(self, i):
        from bitlinear_bl_forward_b200 import bl
        r = i % self.rotations
        if self.one_call:
            bl.bl_forward_norm_grouped([(d["X"], *d["copies"][r], d["L"].N) for d in self.layers], self.norm,
                                       [d["nw"] for d in self.layers] if self.norm == bl.BL_NORM_RMS else None,
                                       eps=1e-5, bits=self.w.bits, outs=[d["Y"] for d in self.layers],
                                       workspace=self.gws)
            return
        for d in self.layers:
            Wp, gamma = d["copies"][r]
            if self.norm == bl.BL_NORM_RMS:
                bl.bl_forward_rmsnorm(d["X"], Wp, gamma, d["L"].N, self.w.bits, norm_weight=d["nw"], eps=1e-5,
                                      out=d["Y"], workspace=d["ws"])
            else:
                bl.bl_forward_layernorm(d["X"], Wp, gamma, d["L"].N, self.w.bits, eps=1e-5, out=d["Y"],
                                        workspace=d["ws"])


def time_quantize_weights(N=28672, K=8192, reps=5):
    """bl_quantize_weights on a 70B-class layer: GB/s of fp32 weights read
    (offline step, not part of the forward metric)."""
    import torch
    from bitlinear_bl_forward_b200 import bl
    W = torch.randn(N, K, device="cuda") * 0.01
    Wp, g = bl.bl_quantize_weights(W)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        bl.bl_quantize_weights(W)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / reps
    del W, Wp, g
    torch.cuda.empty_cache()
    return {"workload": "quantize_weights_70b", "N": N, "K": K, "ms": ms, "GB/s (fp32 W read)": N * K * 4 / ms / 1e6}


def capture(wl, nsteps, start):
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(nsteps):
                wl.step(start + i)
    torch.cuda.current_stream().wait_stream(s)
    return g


def time_workload(wl, steps, warmup, dist_ctx, sample_clocks=True, chunk=None):
    """Warm up, then time exactly `steps` steps with CUDA events on the
    launching stream around graph replays.  (Event nodes inside a graph cost
    several microseconds each, so the per-launch time is the timed region
    divided by the launches it contains.)"""
    import torch
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    chunk = chunk or min(steps, 64 * wl.rotations // math.gcd(64, wl.rotations))
    chunk = max(1, min(chunk, steps))
    g_main = capture(wl, chunk, 0)
    rem = steps % chunk
    g_rem = capture(wl, rem, (steps // chunk) * chunk) if rem else None
    g_main.replay()        # upload + untimed warm replay
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device()) if sample_clocks else None
    if sampler:
        sampler.__enter__()
    dist_ctx.barrier()
    torch.cuda.synchronize()
    # a bounded device-side delay (~200 us of SM clock cycles) ahead of the
    # start event: the host has queued the graph replays by the time the clock
    # starts, so the timed region holds device work only, not graph submission
    torch.cuda._sleep(DELAY_CYCLES)
    t0.record()
    for _ in range(steps // chunk):
        g_main.replay()
    if g_rem is not None:
        g_rem.replay()
    t1.record()
    torch.cuda.synchronize()
    dist_ctx.barrier()
    if sampler:
        sampler.__exit__()
    ms = dist_ctx.max(t0.elapsed_time(t1))
    return ms, (sampler.summary() if sampler else None)


def time_e2e(wl, steps, warmup, dist_ctx):
    """Same metric through the public API with host buffers.  A step that is
    one grouped call goes through the library's host-buffer entry point,
    recorded once as a CUDA graph (bl_forward_grouped_host_graph) and replayed
    once a step (bl_graph_launch): a copy per distinct input from pinned host
    memory, the grouped forward, a copy per output back.
    Other steps copy the inputs from pinned host memory in one transfer, run
    the library calls and read all outputs back in one transfer (the layers'
    tensors are views of one device buffer each, 128-byte aligned)."""
    import torch
    own = [j for j, d in enumerate(wl.layers) if d["own_x"]]

    def carve(shapes):
        offs, n = [], 0
        for shp in shapes:
            offs.append(n)
            n += (int(np.prod(shp)) + 63) // 64 * 64
        return offs, n

    in_offs, n_in = carve([tuple(wl.layers[j]["X"].shape) for j in own])
    out_offs, n_out = carve([tuple(d["Y"].shape) for d in wl.layers])
    dev_in = torch.zeros(n_in, dtype=torch.bfloat16, device="cuda")
    dev_out = torch.empty(n_out, dtype=torch.bfloat16, device="cuda")
    host_in = torch.zeros(n_in, dtype=torch.bfloat16).pin_memory()
    host_out = torch.empty(n_out, dtype=torch.bfloat16).pin_memory()
    for j, off in zip(own, in_offs):
        d = wl.layers[j]
        shp = tuple(d["X"].shape)
        n = int(np.prod(shp))
        host_in[off:off + n].copy_(torch.from_numpy(d["xb"].reshape(-1).view(np.int16)).view(torch.bfloat16))
        view = dev_in[off:off + n].view(shp)
        for dd in wl.layers:                       # every layer that reads this hidden state
            if dd["X"] is d["X"] and dd is not d:
                dd["X"] = view
        d["X"] = view
    for d, off in zip(wl.layers, out_offs):
        shp = tuple(d["Y"].shape)
        d["Y"] = dev_out[off:off + int(np.prod(shp))].view(shp)
    h2d = sum(int(np.prod(tuple(wl.layers[j]["X"].shape))) * 2 for j in own)
    d2h = sum(d["Y"].numel() * 2 for d in wl.layers)

    if len(wl.groups) == 1 and len(wl.groups[0]) > 1 and wl.fmt == "2bit":
        # one grouped call a step: the library's host-buffer entry point
        # copies the step's inputs in, runs the group and copies the outputs
        # back, all on the stream; recorded as a graph, one replay a step
        from bitlinear_bl_forward_b200 import bl
        gr = wl.groups[0]
        hx, hy = {}, {}
        for j, off in zip(own, in_offs):
            shp = tuple(wl.layers[j]["X"].shape)
            hx[j] = host_in[off:off + int(np.prod(shp))].view(shp)
        for j, d in enumerate(wl.layers):
            hx.setdefault(j, hx[d["L"].x_layer if d["L"].x_layer >= 0 else j])
        for j, (d, off) in enumerate(zip(wl.layers, out_offs)):
            shp = tuple(d["Y"].shape)
            hy[j] = host_out[off:off + int(np.prod(shp))].view(shp)
        calls = [bl.PreparedGroupedHost([(hx[j], *wl.layers[j]["copies"][r], wl.layers[j]["L"].N) for j in gr],
                                        [hy[j] for j in gr], wl.w.bits, graph=True) for r in range(wl.rotations)]

        def one(i):
            calls[i % wl.rotations]()
    else:
        def one(i):
            r = i % wl.rotations
            dev_in.copy_(host_in, non_blocking=True)
            for gi in range(len(wl.groups)):
                wl.run_group(gi, r)
            host_out.copy_(dev_out, non_blocking=True)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        one(i)
    t1.record()
    torch.cuda.synchronize()
    dist_ctx.barrier()
    ms = dist_ctx.max(t0.elapsed_time(t1))
    return ms, h2d, d2h


class DistCtx:
    """One process per GPU (torchrun environment): barrier and max over ranks.
    NCCL on GPUs; ``backend="gloo"`` runs the same logic on CPU processes."""

    def __init__(self, ngpus, backend=None):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend or "nccl"
        self.device = "cuda" if self.backend == "nccl" else "cpu"
        self.dist = None
        if self.device == "cuda":
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if self.device == "cuda" else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v):
        if self.dist is None:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()


def replica_value(work_per_rank, n_ranks, ms_max):
    """Whole-job throughput of N independent replicas: every rank's work over
    the slowest rank's time (weak scaling)."""
    return n_ranks * work_per_rank / (ms_max / 1e3)


def roofline_entry(kind, achieved, peak, unit, traffic):
    return {"bound": kind, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic}


def i8_peak(peaks, n_mma=4096, reps=3):
    """Measured dense kind::i8 peak: the library's tcgen05.mma probe on every
    SM at once (M = 128, N = 256, K = 32 MMAs back to back).  Returns a dict
    with TOPS (2 ops per multiply-accumulate) at the clock it ran, the rate per
    SM per clock and that clock; falls back to 2 x the measured bf16 burst
    GEMM when the probe cannot run."""
    import torch
    from bitlinear_bl_forward_b200 import bl
    try:
        best = None
        for _ in range(reps):
            out = bl.bl_probe_mma_i8(n_mma, 256)
            torch.cuda.synchronize()
            o = out.cpu().numpy().astype(np.float64)
            if (o <= 0).any():
                raise RuntimeError("probe wait gave up")
            macs = 128.0 * 256 * 32 * n_mma
            tops = 2 * macs * o.shape[0] / (o[:, 1].max() * 1e-9) / 1e12
            ent = {"tops": tops, "mac_per_clk_per_sm": float(np.median(macs / o[:, 0])),
                   "sm_ghz": float(np.median(o[:, 0] / o[:, 1])), "sms": int(o.shape[0]),
                   "src": "measured tcgen05 kind::i8 probe (bl_probe_mma_i8)"}
            if best is None or ent["tops"] > best["tops"]:
                best = ent
        return best
    except Exception as e:   # report, then fall back to the bf16 burst figure
        return {"tops": peaks["bf16_tflops"] * INT8_NOMINAL_RATIO, "src": f"2 x bf16 burst ({e})"}


def run_gpu(args):
    import torch
    from bitlinear_bl_forward_b200 import build as blbuild
    from bitlinear_bl_forward_b200 import bl
    blbuild.build()
    bl.lib()
    ctx = DistCtx(args.gpus)
    peaks = load_peaks()
    ipk = i8_peak(peaks)
    name = args.workload
    from bitlinear_bl_forward_b200.inputs import WORKLOADS
    w = WORKLOADS[name]
    decode = w.M <= 2
    # enough rotated weight copies that one rotation is > 2x the 126 MB L2
    wbytes = sum(L.N * L.K // 4 for L in w.layers)
    rot = max(2, min(64, int(math.ceil(256e6 / wbytes))))
    wl = GpuWorkload(name, rot)
    K = args.steps if args.steps is not None else (60000 if decode else 2000)
    Wm = max(3, args.warmup)
    ms, clocks = time_workload(wl, K, Wm, ctx)
    N = ctx.world
    sec = ms / 1e3
    if decode:
        value = replica_value(wl.bytes_per_step * K, N, ms) / 1e9
        unit = "GB/s"
    else:
        value = replica_value(wl.ops_per_step * K, N, ms) / 1e12
        unit = "TOPS"

    # dominant kernel: on the decode path every launch of the step is the
    # GEMV, so its average launch duration is the timed region over the
    # launches in it; on the tensor-core path the step also holds the
    # activation-quantisation kernel, so the figure is a lower bound.
    launches = K * wl.launches_per_step
    per_rank_ms = ms
    if decode:
        achieved = wl.bytes_per_step * K / (per_rank_ms / 1e3) / 1e9
        roof = roofline_entry("hbm", achieved, peaks["hbm_gbs"], "GB/s", ncu_traffic(f"decode:{name}"))
    else:
        achieved = wl.ops_per_step * K / (per_rank_ms / 1e3) / 1e12
        roof = roofline_entry("tensor", achieved, ipk["tops"], "TFLOP/s", ncu_traffic(f"tc:{name}"))
    roof["peak_src"] = peaks["src"] + " hbm copy" if decode else ipk["src"]
    roof["kernel"] = ("bl_decode_kernel" if decode else
                      ("bl_mma_persistent_kernel" if w.M <= 64 else "bl_mma_pair_kernel")
                      + " (+ activation quantisation in the step)")
    roof["kernel_us_avg"] = per_rank_ms * 1e3 / launches

    # end-to-end through the public API with host buffers
    e2e_steps = min(K, 2000 if decode else 200)
    ms_e2e, h2d, d2h = time_e2e(wl, e2e_steps, 3, ctx)
    e2e_val = (N * (wl.bytes_per_step if decode else wl.ops_per_step) * e2e_steps / (ms_e2e / 1e3)
               / (1e9 if decode else 1e12))

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": N, "steps": K, "warmup": Wm,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8", "data": "synthetic (seeded; weights N(0, std) generated on the GPU, activations on the host)",
        "config": {"workload": name, "M": w.M, "layers": [[L.name, L.K, L.N] for L in w.layers], "bits": w.bits,
                   "calls_per_step": [[w.layers[j].name for j in gr] for gr in wl.groups],
                   "parallelism": f"replicas x{N}" if N > 1 else "single GPU",
                   "l2": f"{rot} rotated weight copies ({rot * wbytes / 1e6:.0f} MB, > 126 MB L2)",
                   "timing": "CUDA graph replays, events on the launching stream"},
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": K * wl.launches_per_step,
        "roofline": roof,
        "clocks": clocks,
        "i8_peak": ipk,
    }
    if not args.no_secondary and ctx.world == 1:
        line["secondary"] = secondary(args, ctx, peaks, ipk)
    if ctx.rank == 0 and not args.no_cpu_baseline and ctx.world == 1:
        line["cpu_baseline"] = cpu_baseline(name, budget_s=args.cpu_seconds)
    ctx.close()
    if ctx.rank == 0:
        print(json.dumps(line), flush=True)


def secondary(args, ctx, peaks, ipk):
    """Tensor-core workloads, the 70B decode layer and the fused variants:
    each timed region is about 0.3 s, with clocks sampled during it."""
    import torch
    out = []
    want = set(args.secondary.split(",")) if args.secondary else None
    i8 = ipk["tops"]

    def timed(wl, steps):
        ms, clocks = time_workload(wl, steps, 3, ctx, sample_clocks=True)
        return ms, clocks

    def nsteps(n):
        return args.secondary_steps or n

    for name, steps in (("prefill_2b", 2000), ("layer_70b_m1", 25000), ("layer_70b_m16", 10000),
                        ("layer_70b_m128", 8000), ("layer_70b_m2048", 800), ("a48", 4000)):
        if want and name not in want:
            continue
        from bitlinear_bl_forward_b200.inputs import WORKLOADS
        w = WORKLOADS[name]
        wbytes = sum(L.N * L.K // 4 for L in w.layers)
        rot = max(2, min(64, int(math.ceil(256e6 / wbytes))))
        wl = GpuWorkload(name, rot)
        steps = nsteps(steps)
        ms, clocks = timed(wl, steps)
        sec = ms / 1e3
        gbs = wl.bytes_per_step * steps / sec / 1e9
        tops = wl.ops_per_step * steps / sec / 1e12
        out.append({"workload": name, "M": w.M, "ms_per_step": ms / steps, "GB/s": gbs, "TOPS": tops,
                    "hbm_frac": gbs / peaks["hbm_gbs"], "tensor_frac": tops / i8, "steps": steps,
                    "clocks": clocks})
        del wl
        torch.cuda.empty_cache()
    if not want or "layer_70b_m1_base3" in want:
        # the same 70B-class one-token layer with base-3 weight storage (five
        # weights a byte): compare ms_per_step with layer_70b_m1
        wl = GpuWorkload("layer_70b_m1", 6, fmt="b3")
        steps = nsteps(25000)
        ms, clocks = timed(wl, steps)
        gbs = wl.bytes_per_step * steps / (ms / 1e3) / 1e9
        out.append({"workload": "layer_70b_m1_base3", "M": 1, "ms_per_step": ms / steps, "GB/s": gbs,
                    "hbm_frac": gbs / peaks["hbm_gbs"], "steps": steps, "clocks": clocks,
                    "note": "GB/s of the base-3 bytes (1648 B a row instead of 2048); compare ms_per_step"})
        del wl
        torch.cuda.empty_cache()
    if not want or "ffn_2b_decode" in want:
        # the decode feed-forward chain (up+gate grouped, then down on the fused squared ReLU)
        steps = nsteps(60000)
        wl = FfnWorkload(20)
        ms, clocks = timed(wl, steps)
        gbs = wl.bytes_per_step * steps / (ms / 1e3) / 1e9
        out.append({"workload": "ffn_2b_decode", "M": 1, "ms_per_step": ms / steps, "GB/s": gbs,
                    "hbm_frac": gbs / peaks["hbm_gbs"], "steps": steps, "clocks": clocks,
                    "note": "down input = max(0, gate)^2 * up of the same step, formed in the down kernel"})
        del wl
        torch.cuda.empty_cache()
    if not want or "ffn_prefill_2b" in want:
        # up and gate of one 4096-token hidden state: one grouped call (one
        # activation quantisation, one tensor-core launch over both weight
        # tensors) against two single calls on the same buffers
        steps = nsteps(2000)
        res = {}
        for mode in ("grouped", "two_calls"):
            wl = GpuWorkload("ffn_prefill_2b", 16)
            if mode == "two_calls":
                wl.groups = [[0], [1]]
            ms, clocks = timed(wl, steps)
            res[mode] = (ms / steps, clocks, wl.ops_per_step, wl.bytes_per_step)
            del wl
            torch.cuda.empty_cache()
        ms1, clocks, ops, nbytes = res["grouped"]
        tops = ops / (ms1 / 1e3) / 1e12
        out.append({"workload": "ffn_prefill_2b", "M": 4096, "ms_per_step": ms1, "TOPS": tops,
                    "tensor_frac": tops / i8, "GB/s": nbytes / (ms1 / 1e3) / 1e9,
                    "two_calls_ms_per_step": res["two_calls"][0], "steps": steps, "clocks": clocks,
                    "note": "up+gate sharing X in one grouped call vs two bl_forward calls"})
    for name, base, norm, steps, rot in (("rmsnorm_decode_2b", "decode_2b", 0, 20000, 20),
                                         ("rmsnorm_prefill_2b", "prefill_2b", 0, 1200, 20),
                                         ("layernorm_decode_2b", "decode_2b", 1, 20000, 20),
                                         ("layernorm_prefill_2b", "prefill_2b", 1, 1200, 20)):
        if want and name not in want:
            continue
        # the same layers with RMSNorm (bf16 weight) or LayerNorm formed ahead of the quantiser
        wl = NormWorkload(base, rot, norm)
        steps = nsteps(steps)
        ms, clocks = timed(wl, steps)
        sec = ms / 1e3
        gbs = wl.bytes_per_step * steps / sec / 1e9
        ent = {"workload": name, "M": wl.w.M, "ms_per_step": ms / steps, "GB/s": gbs,
               "hbm_frac": gbs / peaks["hbm_gbs"], "steps": steps, "clocks": clocks,
               "note": ("one bl_forward_norm_grouped call over the three layers (one launch)" if wl.w.M == 1 else
                        "one normalised forward call per layer") + ("; norm weight read counted" if norm == 0 else "")}
        if wl.w.M > 1:
            tops = wl.ops_per_step * steps / sec / 1e12
            ent["TOPS"] = tops
            ent["tensor_frac"] = tops / i8
        out.append(ent)
        del wl
        torch.cuda.empty_cache()
    if not want or "quantize_weights_70b" in want:
        out.append(time_quantize_weights())
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_2b")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--secondary", default="", help="comma list restricting the secondary workloads")
    ap.add_argument("--secondary-steps", type=int, default=0,
                    help="timed steps of every secondary line (default: each line's own, about 0.3 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    args = ap.parse_args()
    if args.impl == "reference":
        if args.steps is None:
            args.steps = 20
        run_reference(args)
        return
    run_gpu(args)


if __name__ == "__main__":
    main()
