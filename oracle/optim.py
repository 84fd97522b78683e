"""CPU oracle of the LoRA optimizer step: AdamW with decoupled weight decay and
global-norm gradient clipping, in fp64.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the product path never
imports it, and it imports nothing from the product.

Sources: the diycv.top QLoRA walkthrough, "训练" step 6 (the optimizer updates
only the LoRA parameters) and its recipe paragraph (Adam beta2 = 0.999, max
grad norm 0.3, constant learning rate), §4 "Paged Optimizer" (the state is
paged between device and host; the update itself is unchanged).  The pages do
not spell out the update; reading: the usual AdamW (Loshchilov and Hutter,
decoupled weight decay) with bias-corrected moments, the weight decay applied
before the Adam step, and clipping by the global L2 norm of all LoRA gradients
with coefficient min(1, max_norm / (norm + 1e-6)).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

__all__ = ["clip_coefficient", "adamw_step"]


def clip_coefficient(grads: Sequence[np.ndarray], max_norm: float) -> float:
    """min(1, max_norm / (||g||_2 + 1e-6)) over all gradients together."""
    total = math.sqrt(sum(float(np.sum(np.asarray(g, dtype=np.float64) ** 2)) for g in grads))
    return min(1.0, max_norm / (total + 1e-6))


def adamw_step(params: List[np.ndarray], grads: Sequence[np.ndarray], m: List[np.ndarray], v: List[np.ndarray],
               t: int, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float,
               max_grad_norm: Optional[float]) -> None:
    """One step, in place, fp64:
         g <- g * clip;  p <- p (1 - lr wd);  m <- m + (1 - b1)(g - m);
         v <- b2 v + (1 - b2) g^2;
         p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)."""
    c = 1.0 if max_grad_norm is None else clip_coefficient(grads, max_grad_norm)
    bc1 = 1.0 - beta1 ** t
    bc2 = 1.0 - beta2 ** t
    for p, g, mi, vi in zip(params, grads, m, v):
        g = np.asarray(g, dtype=np.float64) * c
        p *= (1.0 - lr * weight_decay)
        mi += (1.0 - beta1) * (g - mi)
        vi *= beta2
        vi += (1.0 - beta2) * g * g
        p -= (lr / bc1) * mi / (np.sqrt(vi) / math.sqrt(bc2) + eps)
