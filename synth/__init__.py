"""Seeded synthetic inputs for the QLoRA frozen-base linear layer.

This module is shared by the CPU oracle, the tests and the benchmark.  It only
draws random numbers and stores them as bf16 tensors; it holds none of the
method's arithmetic (no quantization, no codebook, no matmul).

Workload recipe (QLoRA, "QLoRA: Efficient Finetuning of Quantized LLMs",
method section on the QLoRA linear layer): frozen base weights W are drawn
N(0, 0.02) and stored as bf16 in the out-major layout W^T[o][h]; activations X
and upstream gradients dY are N(0, 1); the LoRA factors L1[h][r] and L2[r][o]
are N(0, 0.01).  The bulk-quantization workload replaces a fraction of the
weight entries by +-8 sigma outliers.

Every draw uses its own torch CPU generator, seeded from (seed, tag), so a
tensor does not depend on which other tensors were drawn before it.
"""
from __future__ import annotations

import zlib

import torch

__all__ = ["weight_t", "activations", "lora_factors", "tensor_seed"]


def tensor_seed(seed: int, tag: str) -> int:
    """Sub-seed of one named tensor: a CRC of the tag mixed with the run seed."""
    return (int(seed) * 0x9E3779B1 + zlib.crc32(tag.encode())) % (2**63 - 1)


def _normal_bf16(shape, std: float, seed: int, tag: str) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(tensor_seed(seed, tag))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def weight_t(o: int, h: int, seed: int = 0, tag: str = "W", std: float = 0.02,
             outlier_frac: float = 0.0) -> torch.Tensor:
    """Frozen base weight stored transposed: bf16 tensor of shape [o][h].

    With ``outlier_frac`` > 0, that fraction of positions (drawn uniformly with
    replacement from the same seeded stream) is set to exactly +-8*std with a
    random sign.
    """
    w = _normal_bf16((o, h), std, seed, tag)
    if outlier_frac > 0.0:
        n = o * h
        k = max(1, int(round(n * outlier_frac)))
        g = torch.Generator(device="cpu")
        g.manual_seed(tensor_seed(seed, tag + "/outliers"))
        pos = torch.randint(0, n, (k,), generator=g, dtype=torch.int64)
        sign = torch.randint(0, 2, (k,), generator=g, dtype=torch.int64) * 2 - 1
        val = (sign.to(torch.float32) * (8.0 * std)).to(torch.bfloat16)
        w.view(-1)[pos] = val
    return w


def activations(m: int, k: int, seed: int = 0, tag: str = "X", std: float = 1.0) -> torch.Tensor:
    """Row-major bf16 activations (or upstream gradients) of shape [m][k], N(0, std)."""
    return _normal_bf16((m, k), std, seed, tag)


def lora_factors(h: int, r: int, o: int, seed: int = 0, std: float = 0.01):
    """LoRA factors L1 [h][r] and L2 [r][o], bf16, N(0, std)."""
    return (_normal_bf16((h, r), std, seed, "L1"),
            _normal_bf16((r, o), std, seed, "L2"))
