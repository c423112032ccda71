"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the quantization method: it only draws
random tensors with the shapes and value distributions of the workloads and
rounds them to BF16.  Both the CUDA path and the CPU oracle consume exactly
the same BF16 bits (the oracle widens them to float32, which is exact).

Workloads (all synthetic; no dataset or trained weight is used):
  * tiny linear layer: X[128, 256] ~ N(0, 1) with two seeded columns scaled by
    20, W[256, 256] ~ N(0, 0.02^2), dY[128, 256] ~ N(0, (1e-3)^2);
  * Llama-7B-shaped linear layers, tokens M = 32768 (batch 64 x seq 512):
    X[M, K] ~ N(0, 1) except 1% of the K channels drawn from Student-t(3),
    W[N, K] ~ N(0, 0.02^2), dY[M, N] ~ N(0, (1e-3)^2);
  * quantizer sweep: 2^n elements shaped [2^n / 4096, 4096], N(0, 1) with a
    Bernoulli(0.001) subset multiplied by 100;
  * SwiGLU stack: hidden 2048, FFN 8192, tokens 16384, W ~ N(0, 0.02^2).
"""
from __future__ import annotations

import numpy as np
import torch

LLAMA7B_TOKENS = 32768
LLAMA7B_SHAPES = {          # name: (N out-features, K in-features, count per block)
    "qkvo": (4096, 4096, 4),
    "gate_up": (11008, 4096, 2),
    "down": (4096, 11008, 1),
}


def _rng(seed: int, salt: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(salt)]))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy -> BF16 torch CPU tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def as_f32(t: torch.Tensor) -> np.ndarray:
    """BF16 torch tensor -> float32 numpy (exact widening)."""
    return t.detach().to("cpu").float().numpy()


def normal(shape, std: float, seed: int, salt: int = 0) -> torch.Tensor:
    a = _rng(seed, salt).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16(a)


def outlier_columns(M: int, K: int, seed: int, ncols: int = 2, factor: float = 20.0,
                    salt: int = 1):
    """N(0,1) activations with `ncols` seeded columns multiplied by `factor`."""
    rng = _rng(seed, salt)
    a = rng.standard_normal(size=(M, K), dtype=np.float32)
    cols = np.sort(rng.choice(K, size=ncols, replace=False))
    a[:, cols] *= np.float32(factor)
    return to_bf16(a), cols


def student_t_channels(M: int, K: int, seed: int, frac: float = 0.01, df: float = 3.0,
                       salt: int = 2):
    """N(0,1) activations where round(frac*K) seeded channels are Student-t(df)."""
    rng = _rng(seed, salt)
    a = rng.standard_normal(size=(M, K), dtype=np.float32)
    nch = max(1, int(round(frac * K)))
    cols = np.sort(rng.choice(K, size=nch, replace=False))
    a[:, cols] = rng.standard_t(df, size=(M, nch)).astype(np.float32)
    return to_bf16(a), cols


def sparse_outliers(rows: int, cols: int, seed: int, p: float = 1e-3, factor: float = 100.0,
                    salt: int = 3):
    """N(0,1) with a Bernoulli(p) subset of elements multiplied by `factor`."""
    rng = _rng(seed, salt)
    a = rng.standard_normal(size=(rows, cols), dtype=np.float32)
    mask = rng.random(size=(rows, cols), dtype=np.float32) < p
    a[mask] *= np.float32(factor)
    return to_bf16(a)


def tiny_linear(seed: int = 0) -> dict:
    X, cols = outlier_columns(128, 256, seed)
    return {"X": X, "W": normal((256, 256), 0.02, seed, 10),
            "dY": normal((128, 256), 1e-3, seed, 11), "outlier_cols": cols}


def llama_linear(N: int, K: int, M: int = LLAMA7B_TOKENS, seed: int = 0) -> dict:
    X, cols = student_t_channels(M, K, seed, salt=100 + K)
    return {"X": X, "W": normal((N, K), 0.02, seed, 200 + N * 7 + K),
            "dY": normal((M, N), 1e-3, seed, 300 + N), "t_channels": cols}


def sweep_tensor(log2_n: int, seed: int = 0, width: int = 4096) -> torch.Tensor:
    n = 1 << log2_n
    return sparse_outliers(max(1, n // width), min(n, width), seed)
