"""Data-parallel exchange for the QLoRA linear layer.

The pages note that QLoRA training scales out with ordinary data parallelism
(robocikowo.com QLoRA glossary, parallelism entry: DDP / FSDP).  With the base
weight frozen, every rank holds the same NF4 weight, runs the layer on its own
tokens, and the only exchange is the sum of the LoRA gradients dL1 and dL2
over ranks: one all-reduce of (h + o) * r fp32 values per layer.

The gradients are allocated as two views of one flat buffer, so the exchange is
a single collective with no packing copies.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def lora_grad_buffers(h: int, o: int, r: int, device, dtype=torch.float32
                      ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """One flat fp32 buffer and its two views dL1 [h][r], dL2 [r][o]."""
    flat = torch.empty(h * r + r * o, dtype=dtype, device=device)
    dL1 = flat[: h * r].view(h, r)
    dL2 = flat[h * r:].view(r, o)
    return flat, dL1, dL2


def allreduce_lora_grads(flat: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> None:
    """Sums the packed LoRA gradients over the data-parallel group, in place."""
    if not dist.is_available() or not dist.is_initialized():
        return
    if dist.get_world_size(group) == 1:
        return
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)


def shard_rows(M: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous token range [begin, end) of one rank (sizes differ by at most 1)."""
    base, extra = divmod(M, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)
