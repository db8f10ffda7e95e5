"""Seeded synthetic inputs shared by the tests, the smoke check and bench.py.

This module holds no quantization or GEMM arithmetic: it only draws random
numbers (numpy PCG64) and rounds them to bf16.  The same bf16 bytes feed the
CPU oracle and the CUDA library.

Workloads (each a stand-in for the shapes and value distributions the pages
discuss; no dataset is used):
  pr1_tiny       M=16, K=256, N=256; A ~ N(0,1) with 1% of entries set to
                 +-1000; W ~ N(0, 0.02)                                (seed 0)
  act_sweep      x[m,k] = z * exp(u_m), z ~ N(0,1), u_m ~ N(0,1) per row
                 (per-row lognormal scale, sigma = 1)                  (seed 1)
  decode         A ~ N(0,1), W ~ N(0, 0.02)                            (seed 2)
  prefill        A ~ N(0,1) with 0.1% of entries multiplied by 100;
                 W ~ N(0, 0.02)                                        (seed 3)
  decoder        24-layer synthetic decoder weights ~ N(0, 0.02)       (seed 4)
"""
from __future__ import annotations

import numpy as np
import torch

SEED_PR1, SEED_ACT, SEED_DECODE, SEED_PREFILL, SEED_DECODER = 0, 1, 2, 3, 4


def rng(seed: int, *shape_tag: int) -> np.random.Generator:
    """A PCG64 generator keyed by the workload seed and the shape."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *shape_tag])))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy -> bf16 torch tensor on the CPU (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def pr1_tiny():
    """A [16,256] with 41 (= 1% of 4096) +-1000 outliers, W [256,256]."""
    g = rng(SEED_PR1, 16, 256, 256)
    a = normal(g, (16, 256))
    n_out = int(round(0.01 * a.size))
    pos = g.choice(a.size, size=n_out, replace=False)
    sign = np.where(g.integers(0, 2, size=n_out) == 0, -1.0, 1.0).astype(np.float32)
    a.reshape(-1)[pos] = sign * np.float32(1000.0)
    w = normal(g, (256, 256), 0.02)
    return to_bf16(a), to_bf16(w)


def act_sweep(M: int, K: int):
    """Activation-quantize workload: per-row lognormal-scaled normals."""
    g = rng(SEED_ACT, M, K)
    u = g.standard_normal(size=(M, 1), dtype=np.float32)
    z = normal(g, (M, K))
    return to_bf16(z * np.exp(u))


def decode(M: int, N: int, K: int):
    g = rng(SEED_DECODE, M, N, K)
    a = normal(g, (M, K))
    w = normal(g, (N, K), 0.02)
    return to_bf16(a), to_bf16(w)


def prefill(M: int, N: int, K: int):
    """A with round(0.1% * M * K) entries multiplied by 100; W ~ N(0, 0.02)."""
    g = rng(SEED_PREFILL, M, N, K)
    a = normal(g, (M, K))
    n_out = int(round(0.001 * a.size))
    pos = g.choice(a.size, size=n_out, replace=False)
    a.reshape(-1)[pos] *= np.float32(100.0)
    w = normal(g, (N, K), 0.02)
    return to_bf16(a), to_bf16(w)


def random_bf16(seed: int, shape, std: float = 1.0):
    g = rng(seed, *shape)
    return to_bf16(normal(g, shape, std))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy array of its bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
