"""Shared helpers for the GPU parity tests (host <-> device marshalling and the
comparison rules).  The CUDA side is reached only through the C ABI binding;
the expected values come only from the oracle."""

from __future__ import annotations

import numpy as np
import torch


def x_to_dev(x_bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> bf16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_dev_to_bits(y: torch.Tensor) -> np.ndarray:
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns
    (monotone integer mapping of the sign-magnitude encoding)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + (b & 0x7FFF))
    return np.abs(key(a_bits) - key(b_bits))


def rel_err(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    want = want.astype(np.float64)
    d = np.abs(got.astype(np.float64) - want)
    return np.where(want != 0, d / np.maximum(np.abs(want), 1e-300), d)


# Tolerances (stated with the target): fp32 output within 1e-3 relative of the
# oracle; bf16 output within 1 ulp of the oracle's fp32 value rounded to bf16.
F32_REL_TOL = 1e-3
BF16_ULP_TOL = 1
