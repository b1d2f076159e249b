"""Seeded synthetic inputs for the QLoRA frozen-base linear layer.

This module only draws random tensors; it holds none of the quantizer's,
dequantizer's or the layer's arithmetic. Both the CPU oracle (tests) and
the CUDA path (tests, benchmark) take their inputs from here, so the two
sides always see identical bytes.

Distributions follow the workloads of "QLoRA Explained: Fine-Tune 70B+ LLMs
on a Single GPU" and "QLoRA: Quantized Low-Rank Adaptation" (frozen weights
that are roughly normal with zero mean, section "NF4: a 4-bit format matched
to weight statistics"):

* W  ~ N(0, 0.02^2), fp32, optionally with a fraction of outliers at
  +/- 10 sigma (indices uniform without replacement, sign uniform);
* X, dY ~ N(0, 1), rounded to bf16 (round-to-nearest-even, torch CPU cast);
* A ~ N(0, (1/r)^2), B ~ N(0, 0.01^2), rounded to bf16 (B non-zero on purpose
  so that the low-rank branch of the forward pass and dA are exercised).

N(mean, s) is read as (mean, standard deviation) throughout.

All generators use torch's CPU generator with fixed seeds; for a stack of
layers the seed is offset by 100 per layer index.
"""
from __future__ import annotations

import torch

SEED_W, SEED_X, SEED_A, SEED_B, SEED_DY, SEED_OUTLIER = 1, 2, 3, 4, 5, 6
LAYER_SEED_STRIDE = 100


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(n: int, k: int, std: float = 0.02, outlier_frac: float = 0.0,
           outlier_sigma: float = 10.0, layer: int = 0) -> torch.Tensor:
    """fp32 [n, k] weight matrix, row-major (out_features x in_features)."""
    off = LAYER_SEED_STRIDE * layer
    w = torch.randn(n, k, generator=_gen(SEED_W + off), dtype=torch.float32) * std
    if outlier_frac > 0.0:
        count = int(round(outlier_frac * n * k))
        g = _gen(SEED_OUTLIER + off)
        idx = torch.randperm(n * k, generator=g)[:count]
        sign = torch.randint(0, 2, (count,), generator=g, dtype=torch.int64) * 2 - 1
        w.view(-1)[idx] = sign.to(torch.float32) * (outlier_sigma * std)
    return w.contiguous()


def activations(m: int, k: int, layer: int = 0, seed: int = SEED_X) -> torch.Tensor:
    """bf16 [m, k] activations ~ N(0, 1)."""
    off = LAYER_SEED_STRIDE * layer
    x = torch.randn(m, k, generator=_gen(seed + off), dtype=torch.float32)
    return x.to(torch.bfloat16).contiguous()


def grad_output(m: int, n: int, layer: int = 0) -> torch.Tensor:
    """bf16 [m, n] upstream gradient dY ~ N(0, 1)."""
    return activations(m, n, layer=layer, seed=SEED_DY)


def lora_pair(r: int, k: int, n: int, layer: int = 0):
    """bf16 adapters A [r, k] ~ N(0, (1/r)^2) and B [n, r] ~ N(0, 0.01^2)."""
    off = LAYER_SEED_STRIDE * layer
    a = torch.randn(r, k, generator=_gen(SEED_A + off), dtype=torch.float32) * (1.0 / r)
    b = torch.randn(n, r, generator=_gen(SEED_B + off), dtype=torch.float32) * 0.01
    return a.to(torch.bfloat16).contiguous(), b.to(torch.bfloat16).contiguous()


def sample_rows(m: int, count: int, seed: int = 7) -> torch.Tensor:
    """Sorted distinct row indices in [0, m) for sampled comparisons."""
    count = min(count, m)
    return torch.sort(torch.randperm(m, generator=_gen(seed))[:count]).values
