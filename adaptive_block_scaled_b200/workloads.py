"""Seeded synthetic inputs shaped like the workloads the IF4 pages evaluate on.

This module only draws random numbers and casts them; it holds none of the
IF4 arithmetic.  The tests feed the same tensors to the CUDA path and to the
CPU oracle, and the benchmark times the CUDA path on them.

The pages evaluate on LLM weights, activations and Hadamard-transformed weight
gradients (episode companion "Adaptive Block-Scaled Data Types for FP4
Training", sections "Training Loss vs. BF16 Baseline" and "Where the Gain
Actually Comes From"; gist.science section 1 on the Hadamard transform).  No
checkpoints or datasets are used: each recipe below draws a stand-in with the
named distribution from ``numpy.random.default_rng(seed)`` (PCG64), in
float32, then casts to bfloat16 by round-to-nearest-even (torch CPU cast).
"""
from dataclasses import dataclass

import numpy as np
import torch


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def small_fp32(seed: int = 0, rows: int = 256, cols: int = 1024) -> torch.Tensor:
    """float32 [rows, cols], i.i.d. N(0, 1)."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((rows, cols), dtype=np.float32))


def llm_weight(seed: int = 0, rows: int = 4096, cols: int = 4096, std: float = 0.02) -> torch.Tensor:
    """bfloat16 [N, K] weight: Student-t (nu = 3) draws rescaled to std ``std``
    (a t(3) variable has variance 3)."""
    rng = np.random.default_rng(seed)
    t = rng.standard_t(3, size=(rows, cols))
    return _bf16(t * (std / np.sqrt(3.0)))


def activation_outliers(seed: int = 0, tokens: int = 8192, hidden: int = 8192,
                        outlier_frac: float = 0.01, gain: float = 20.0) -> torch.Tensor:
    """bfloat16 [tokens, hidden] activations: N(0, 1) with round(1% of hidden)
    channels, fixed by the seed, multiplied by ``gain``."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((tokens, hidden), dtype=np.float32)
    n_out = int(round(outlier_frac * hidden))
    ch = rng.choice(hidden, n_out, replace=False)
    x[:, ch] *= np.float32(gain)
    return _bf16(x)


def sylvester_hadamard(n: int = 16) -> np.ndarray:
    h = np.ones((1, 1), np.float32)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_gradient(seed: int = 0, rows: int = 16384, cols: int = 4096,
                      std: float = 1e-3) -> torch.Tensor:
    """bfloat16 [rows, cols] gradient-like tensor: N(0, std) draws, then, inside
    every 16-element group along the row, y = H16 diag(s) x / 4 with H16 the
    Sylvester Hadamard matrix and s one seeded +-1 vector shared by all groups
    (an orthonormal random-sign Hadamard transform), computed in float32."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    s = rng.choice(np.array([-1.0, 1.0], np.float32), 16)
    m = (sylvester_hadamard(16) * s[None, :]) / np.float32(4.0)
    y = (x.reshape(-1, 16) @ m.T.astype(np.float32)).reshape(rows, cols)
    return _bf16(y)


def linear_operands(seed: int = 0, M: int = 8192, N: int = 4096, K: int = 4096,
                    b_std: float = 0.02):
    """A = N(0, 1) [M, K] activations, then B = N(0, b_std) [N, K] weights, both
    bfloat16, drawn from one generator in that order."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    b = rng.standard_normal((N, K), dtype=np.float32) * np.float32(b_std)
    return _bf16(a), _bf16(b)


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    make: object          # callable(seed) -> tensor, or (A, B) for the linear
    shape: tuple


WORKLOADS = {
    "small_fp32_256x1024": Workload(
        "small_fp32_256x1024", "float32 256x1024, N(0,1), groups of 16 along rows",
        small_fp32, (256, 1024)),
    "weight_bf16_4096x4096": Workload(
        "weight_bf16_4096x4096",
        "LLM weight bf16 4096x4096, Student-t(3) scaled to std 0.02, groups of 16 along K",
        llm_weight, (4096, 4096)),
    "activation_bf16_8192x8192": Workload(
        "activation_bf16_8192x8192",
        "activations bf16 8192 tokens x 8192 hidden, N(0,1), 1% of channels x20",
        activation_outliers, (8192, 8192)),
    "gradient_bf16_16384x4096": Workload(
        "gradient_bf16_16384x4096",
        "weight-gradient-like bf16 16384x4096, N(0,1e-3) then random-sign 16-point Hadamard per group",
        hadamard_gradient, (16384, 4096)),
    "linear_8192x4096x4096": Workload(
        "linear_8192x4096x4096",
        "IF4xIF4 linear: A bf16 8192x4096 N(0,1), B bf16 4096x4096 N(0,0.02), IF4 along K",
        linear_operands, (8192, 4096, 4096)),
}
