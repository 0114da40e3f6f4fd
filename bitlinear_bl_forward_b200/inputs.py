"""Seeded synthetic inputs shaped like the layers the pages discuss.

This module only draws random numbers; it holds none of the BitLinear
arithmetic.  Both the CUDA-path tests/benchmark and the CPU oracle consume the
same arrays, generated on the host with torch's CPU generator so that every
run, on any machine with or without a GPU, sees identical bits.

Recipe (per workload; ``seed`` defaults to 0):
  * weights:  W fp32 [N, K] = std * N(0, 1), generator seed = seed + 10*i for
    the i-th layer of the workload;
  * activations: X [M, K] drawn in fp32 from N(0, 1) with generator seed
    seed + 1 + 10*i (i = the layer whose input it is: up and gate of a
    feed-forward block share one), then
      - "outliers": n_out channels (columns) chosen by randperm(K) with seed
        seed + 2 + 10*i are multiplied by ``mult`` for every token,
      - "relu2":    X = max(0, z)^2 elementwise,
      - "normal":   unchanged;
    and finally rounded to bf16 (round to nearest even).  X is returned as
    bf16 bit patterns (uint16).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Layer:
    name: str
    K: int          # in-features
    N: int          # out-features
    x_layer: int = -1   # >= 0: this layer reads the activations of that layer (same hidden state)


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    layers: tuple
    w_std: float
    x_kind: str                 # "outliers" | "normal" | "relu2"
    n_outliers: object = 0      # int, or "1%" meaning round(0.01*K)
    outlier_mult: float = 1.0
    bits: int = 8
    note: str = ""
    groups: tuple = ()          # layers a step runs in one grouped call, e.g. ((0, 1, 2),)

    def outliers_for(self, K: int) -> int:
        if isinstance(self.n_outliers, str) and self.n_outliers.endswith("%"):
            return int(round(float(self.n_outliers[:-1]) / 100.0 * K))
        return int(self.n_outliers)


# The five workloads (shapes and distributions of the 2B- and 70B-class
# layers, plus the 4-bit-activation a4.8 layer).
WORKLOADS = {
    "tiny": Workload("tiny", 16, (Layer("proj", 256, 512),), 0.02, "outliers", 2, 20.0, 8,
                     "tiny BitLinear 16x256 -> 512"),
    # up and gate project the same hidden state; down reads its own input
    "decode_2b": Workload("decode_2b", 1,
                          (Layer("up", 2560, 6912), Layer("gate", 2560, 6912, x_layer=0), Layer("down", 6912, 2560)),
                          0.02, "outliers", "1%", 10.0, 8, "2B-class decode GEMV, batch 1", ((0, 1, 2),)),
    "prefill_2b": Workload("prefill_2b", 4096,
                           (Layer("up", 2560, 6912), Layer("down", 6912, 2560)),
                           0.02, "outliers", "1%", 10.0, 8, "2B-class prefill GEMM, 4096 tokens"),
    "layer_70b_m1": Workload("layer_70b_m1", 1, (Layer("ffn", 8192, 28672),), 0.01, "normal", 0, 1.0, 8,
                             "70B-class layer, M=1"),
    "layer_70b_m16": Workload("layer_70b_m16", 16, (Layer("ffn", 8192, 28672),), 0.01, "normal", 0, 1.0, 8,
                              "70B-class layer, M=16"),
    "layer_70b_m128": Workload("layer_70b_m128", 128, (Layer("ffn", 8192, 28672),), 0.01, "normal", 0, 1.0, 8,
                               "70B-class layer, M=128"),
    "layer_70b_m2048": Workload("layer_70b_m2048", 2048, (Layer("ffn", 8192, 28672),), 0.01, "normal", 0, 1.0, 8,
                                "70B-class layer, M=2048"),
    "a48": Workload("a48", 2048, (Layer("proj", 4096, 11008),), 0.02, "relu2", 0, 1.0, 4,
                    "a4.8 mode: 4-bit activations, 2048x4096 -> 11008"),
    # the 2B prefill feed-forward input side: up and gate of one hidden state
    "ffn_prefill_2b": Workload("ffn_prefill_2b", 4096, (Layer("up", 2560, 6912), Layer("gate", 2560, 6912, x_layer=0)),
                               0.02, "outliers", "1%", 10.0, 8, "2B-class up+gate prefill, 4096 tokens", ((0, 1),)),
}


def make_weight(N: int, K: int, std: float, seed: int) -> np.ndarray:
    g = torch.Generator().manual_seed(int(seed))
    return (torch.randn(N, K, generator=g, dtype=torch.float32) * std).numpy()


def make_activation(M: int, K: int, kind: str, seed: int, n_outliers: int = 0,
                    mult: float = 1.0) -> np.ndarray:
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if kind == "outliers" and n_outliers > 0:
        g2 = torch.Generator().manual_seed(int(seed) + 1)
        ch = torch.randperm(K, generator=g2)[:n_outliers]
        x[:, ch] *= mult
    elif kind == "relu2":
        x = torch.relu(x) ** 2
    elif kind not in ("normal", "outliers"):
        raise ValueError(kind)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def layer_inputs(w: Workload, i: int, seed: int = 0, M: int | None = None):
    """(X bf16 bits [M, K], W fp32 [N, K]) for layer i of workload w."""
    L = w.layers[i]
    M = w.M if M is None else M
    W = make_weight(L.N, L.K, w.w_std, seed + 10 * i)
    xi = i if L.x_layer < 0 else L.x_layer
    X = make_activation(M, L.K, w.x_kind, seed + 1 + 10 * xi, w.outliers_for(L.K), w.outlier_mult)
    return X, W


def random_case(M: int, K: int, N: int, seed: int, w_std: float = 0.02,
                x_kind: str = "outliers", n_outliers: int = 2, mult: float = 20.0):
    """A small seeded case with arbitrary shape (used for ragged-shape tests)."""
    W = make_weight(N, K, w_std, seed)
    X = make_activation(M, K, x_kind, seed + 1, min(n_outliers, K), mult)
    return X, W
