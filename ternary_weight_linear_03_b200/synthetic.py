"""Seeded synthetic inputs shaped like the BitLinear workloads.

This module only draws random numbers; it holds none of the method's arithmetic, so
both the CUDA path and the oracle may take their inputs from it.

Recipe (every tensor is drawn on the CPU with ``torch.Generator().manual_seed(seed)``):
  * weights: ``randn(N, K) * sigma`` in fp32 (sigma 0.02 for the 700M/3B-class shapes,
    0.015 for the 70B-class shapes);
  * activations: ``randn(M, K)`` in fp32; with ``outlier_frac > 0`` a seeded choice of
    ceil(outlier_frac * K) channels (the same channels for every token) is multiplied by
    ``outlier_gain``; then cast to bf16 where the workload says bf16.
"""

from __future__ import annotations

import math

import torch


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, sigma: float, seed: int, dtype=torch.float32,
            device="cpu") -> torch.Tensor:
    """N x K weights ~ N(0, sigma^2). device="cpu" is the reference recipe (CPU generator,
    what the parity tests use); a CUDA device draws the same distribution with that
    device's seeded generator (other values, far faster for the large benchmark sets)."""
    w = torch.randn((N, K), generator=gen(seed, device), dtype=torch.float32, device=device)
    w.mul_(sigma)
    return w.to(dtype)


def activations(M: int, K: int, seed: int, dtype=torch.bfloat16, outlier_frac: float = 0.0,
                outlier_gain: float = 20.0, device="cpu") -> torch.Tensor:
    g = gen(seed, device)
    x = torch.randn((M, K), generator=g, dtype=torch.float32, device=device)
    if outlier_frac > 0.0:
        n_out = int(math.ceil(outlier_frac * K))
        cols = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, cols] *= outlier_gain
    return x.to(dtype)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (the oracle's bf16 input form)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")


# Workloads: (name, N, K, sigma, M list, x dtype, outliers)
WORKLOADS = {
    "tiny_256x256": dict(N=256, K=256, sigma=0.02, Ms=[8], x_dtype=torch.float32,
                         outlier_frac=0.0, w_seed=0, x_seed=0),
    "700m_up_1536x4096": dict(N=4096, K=1536, sigma=0.02, Ms=[1, 4, 16],
                              x_dtype=torch.bfloat16, outlier_frac=0.01),
    "3b_gate_up_3200x8640": dict(N=8640, K=3200, sigma=0.02, Ms=[1, 16, 64],
                                 x_dtype=torch.bfloat16, outlier_frac=0.0),
    "3b_down_8640x3200": dict(N=3200, K=8640, sigma=0.02, Ms=[1, 16, 64],
                              x_dtype=torch.bfloat16, outlier_frac=0.0),
    "70b_up_8192x28672": dict(N=28672, K=8192, sigma=0.015, Ms=[1, 16, 176],
                              x_dtype=torch.bfloat16, outlier_frac=0.0),
    "70b_down_28672x8192": dict(N=8192, K=28672, sigma=0.015, Ms=[1, 16, 176],
                                x_dtype=torch.bfloat16, outlier_frac=0.0),
    "70b_prefill_4096x8192x28672": dict(N=28672, K=8192, sigma=0.015, Ms=[4096],
                                        x_dtype=torch.bfloat16, outlier_frac=0.0),
}


def w_seed(name: str, matrix_index: int = 0) -> int:
    wl = WORKLOADS[name]
    return wl.get("w_seed", 1000 + matrix_index)


def x_seed(name: str, M: int) -> int:
    wl = WORKLOADS[name]
    return wl.get("x_seed", 2000 + M)
