"""Token-sharded data parallelism for the QLoRA frozen-base linear layer.

The layer shards naturally by tokens ("QLoRA Explained: Fine-Tune 70B+ LLMs on
a Single GPU", Hardware Requirements by Model Size and the VRAM FAQ on running
one model over several GPUs): every rank holds the same NF4 weight and the same
adapters A, B, and processes its own contiguous slice of the tokens.

* Forward: Y and U of a rank's tokens depend only on those tokens; no exchange.
* Backward: dX of a rank's tokens is local too. The adapter gradients are sums
  over tokens, dA = s G^T X and dB = s dY^T U, so each rank's call of
  qlora_linear_bwd on its slice yields a partial sum, and the full-batch
  gradient is the sum over ranks: one all-reduce (sum) of dA and dB per step.

This module is host plumbing only (torch.distributed: NCCL between GPUs, gloo
on CPU); it holds none of the layer's arithmetic. Gradients of all layers live
in one flat fp32 buffer so that the exchange is a single collective.
"""
from __future__ import annotations

from typing import Dict, Iterable, Tuple

import torch
import torch.distributed as dist


def world() -> Tuple[int, int]:
    """(rank, world size) of the initialised process group, else (0, 1)."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def token_shard(m_total: int, rank: int, world_size: int) -> Tuple[int, int]:
    """Contiguous token range [start, stop) of `rank` when m_total tokens are split
    over world_size ranks; the first m_total % world_size ranks get one more."""
    if world_size < 1 or not 0 <= rank < world_size or m_total < 0:
        raise ValueError("need 0 <= rank < world_size and m_total >= 0")
    base, extra = divmod(m_total, world_size)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class AdapterGrads:
    """fp32 dA [r, k] and dB [n, r] of several layers as views of one flat buffer.

    layers: iterable of (name, n, k); r is the LoRA rank. `dA[name]` and
    `dB[name]` are the tensors to pass to qlora_linear_bwd; `all_reduce()` sums
    every layer's gradients over the ranks in one collective."""

    def __init__(self, layers: Iterable[Tuple[str, int, int]], r: int, device=None):
        layers = list(layers)
        sizes = [r * k + n * r for _, n, k in layers]
        self.flat = torch.zeros(sum(sizes), dtype=torch.float32, device=device)
        self.dA: Dict[str, torch.Tensor] = {}
        self.dB: Dict[str, torch.Tensor] = {}
        off = 0
        for (name, n, k), size in zip(layers, sizes):
            self.dA[name] = self.flat[off:off + r * k].view(r, k)
            self.dB[name] = self.flat[off + r * k:off + size].view(n, r)
            off += size

    def zero_(self) -> None:
        self.flat.zero_()

    def all_reduce(self) -> None:
        all_reduce_sum(self.flat)


def all_reduce_sum(flat: torch.Tensor) -> None:
    """Sum `flat` over all ranks in place (no-op without a process group or with one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)


def max_over_ranks(x: float) -> float:
    """Largest value of x over the ranks (the step time of a data-parallel job)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
