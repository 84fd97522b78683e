"""Paged AdamW for the LoRA factors (the paged optimizer of QLoRA: optimizer
state in NVIDIA unified memory that moves to host RAM under memory pressure
and back when the update needs it).

The arithmetic runs in libqlora.so (qlora_grad_sqnorm, qlora_adamw_step); the
state lives in unified memory from qlora_paged_alloc, placed with
qlora_paged_advise / qlora_paged_prefetch.  This module only holds buffers and
the host-side policy that decides when to move the state: before a step the
state is brought back to the device if there is room for it, and when free
device memory falls below a watermark (a spike) it is sent to host RAM.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple

import torch

from ._lib import _check, _stream, lib, qlora_adamw_t


class ManagedBuffer:
    """An fp32 array in unified memory, usable as a CUDA torch tensor (a view
    through __cuda_array_interface__; the buffer owns the memory)."""

    def __init__(self, numel: int, device: torch.device):
        self.numel = int(numel)
        self.nbytes = 4 * self.numel
        self.device = torch.device(device)
        ptr = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib().qlora_paged_alloc(self.nbytes, ctypes.byref(ptr)), "qlora_paged_alloc")
        self.ptr = int(ptr.value)
        self.__cuda_array_interface__ = {"shape": (self.numel,), "typestr": "<f4", "data": (self.ptr, False),
                                         "version": 3, "strides": None}
        with torch.cuda.device(self.device):
            self.tensor = torch.as_tensor(self, device=self.device)

    def advise(self, prefer_host: bool) -> None:
        with torch.cuda.device(self.device):
            _check(lib().qlora_paged_advise(ctypes.c_void_p(self.ptr), self.nbytes, 1 if prefer_host else 0),
                   "qlora_paged_advise")

    def prefetch(self, to_host: bool) -> None:
        with torch.cuda.device(self.device):
            _check(lib().qlora_paged_prefetch(ctypes.c_void_p(self.ptr), self.nbytes, 1 if to_host else 0,
                                              _stream(self.device)), "qlora_paged_prefetch")

    def free(self) -> None:
        if self.ptr:
            self.tensor = None
            torch.cuda.synchronize(self.device)
            _check(lib().qlora_paged_free(ctypes.c_void_p(self.ptr)), "qlora_paged_free")
            self.ptr = 0

    def __del__(self):
        try:
            self.free()
        except Exception:  # noqa: BLE001  (interpreter shutdown)
            pass


class PagingPolicy:
    """When to move the optimizer state (host logic only, testable on a CPU
    with a fake memory probe and a fake mover).

    mem_info() returns (free, total) device bytes.  on_step() is called before
    each update: state on the host comes back if the device then keeps at least
    `watermark` bytes free.  on_pressure() is called when a memory spike may be
    coming (e.g. after the forward of a long sequence): if free memory is below
    `watermark`, state on the device goes to the host.  move(to_host) performs
    the move and the policy records where the state is."""

    def __init__(self, state_bytes: int, watermark: int, mem_info: Callable[[], Tuple[int, int]],
                 move: Callable[[bool], None]):
        self.state_bytes = int(state_bytes)
        self.watermark = int(watermark)
        self.mem_info = mem_info
        self.move = move
        self.on_host = False
        self.moves: List[str] = []

    def on_pressure(self) -> bool:
        free, _ = self.mem_info()
        if not self.on_host and free < self.watermark:
            self.move(True)
            self.on_host = True
            self.moves.append("to_host")
            return True
        return False

    def on_step(self) -> bool:
        free, _ = self.mem_info()
        if self.on_host and free - self.state_bytes >= self.watermark:
            self.move(False)
            self.on_host = False
            self.moves.append("to_device")
            return True
        return False


@dataclass
class AdamWConfig:
    """AdamW hyper-parameters; the defaults follow the QLoRA recipe (Adam
    beta2 = 0.999, max grad norm 0.3, constant learning rate)."""
    lr: float = 2e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0
    max_grad_norm: Optional[float] = 0.3


class PagedAdamW:
    """AdamW over the fp32 master copy of all LoRA factors, held as one flat
    buffer (so that a step is two launches whatever the number of layers),
    with its state (m, v) in unified memory.

    param: fp32 CUDA tensor [n], updated in place (views of it are the
    factors); copy (optional): bf16 tensor [n], the adapter weights the layer
    reads, written after each step.  grads passed to step() have the same
    flat layout.  With watermark_bytes > 0 the paging policy probes free
    device memory before each step and on on_pressure()."""

    def __init__(self, param: torch.Tensor, cfg: AdamWConfig = AdamWConfig(), copy: Optional[torch.Tensor] = None,
                 watermark_bytes: int = 0, mem_info: Optional[Callable[[], Tuple[int, int]]] = None):
        if not (param.is_cuda and param.dtype == torch.float32 and param.is_contiguous() and param.dim() == 1):
            raise ValueError("param must be a flat contiguous fp32 CUDA tensor")
        if copy is not None and (copy.dtype != torch.bfloat16 or copy.shape != param.shape or
                                 not copy.is_contiguous() or copy.device != param.device):
            raise ValueError("copy must be a contiguous bf16 tensor shaped like param")
        self.param, self.copy, self.cfg = param, copy, cfg
        self.t = 0
        self.device = param.device
        self.n = param.numel()
        self.m = ManagedBuffer(self.n, self.device)
        self.v = ManagedBuffer(self.n, self.device)
        self.m.tensor.zero_()
        self.v.tensor.zero_()
        self.sqnorm = torch.zeros(1, dtype=torch.float64, device=self.device)
        self.watermark = int(watermark_bytes)
        self.policy = PagingPolicy(self.m.nbytes + self.v.nbytes, self.watermark,
                                   mem_info or (lambda: torch.cuda.mem_get_info(self.device)), self._move)

    def _move(self, to_host: bool) -> None:
        for b in (self.m, self.v):
            b.advise(prefer_host=to_host)
            b.prefetch(to_host=to_host)

    def evict(self) -> None:
        """Send the state to host RAM now (what a memory spike does)."""
        if not self.policy.on_host:
            self._move(True)
            self.policy.on_host = True
            self.policy.moves.append("to_host")

    def step(self, grad: torch.Tensor) -> None:
        if grad.shape != self.param.shape or grad.dtype != torch.float32 or not grad.is_contiguous() or \
                grad.device != self.device:
            raise ValueError("grad must be a flat contiguous fp32 tensor shaped like param")
        if self.watermark > 0 or self.policy.on_host:
            self.policy.on_step()
        self.t += 1
        L = lib()
        st = _stream(self.device)
        clip = self.cfg.max_grad_norm is not None
        hp = qlora_adamw_t(self.cfg.lr, self.cfg.beta1, self.cfg.beta2, self.cfg.eps, self.cfg.weight_decay,
                           float(self.cfg.max_grad_norm or 0.0), self.t)
        with torch.cuda.device(self.device):
            if clip:
                self.sqnorm.zero_()
                _check(L.qlora_grad_sqnorm(ctypes.c_void_p(grad.data_ptr()), self.n,
                                           ctypes.c_void_p(self.sqnorm.data_ptr()), st), "qlora_grad_sqnorm")
            _check(L.qlora_adamw_step(ctypes.c_void_p(self.param.data_ptr()), ctypes.c_void_p(grad.data_ptr()),
                                      ctypes.c_void_p(self.m.ptr), ctypes.c_void_p(self.v.ptr),
                                      ctypes.c_void_p(self.copy.data_ptr()) if self.copy is not None else None,
                                      self.n, ctypes.byref(hp),
                                      ctypes.c_void_p(self.sqnorm.data_ptr()) if clip else None, st),
                   "qlora_adamw_step")

    def close(self) -> None:
        self.m.free()
        self.v.free()


def flat_views(flat: torch.Tensor, shapes: Sequence[Tuple[int, ...]]) -> List[torch.Tensor]:
    """Consecutive views of a flat tensor with the given shapes (e.g. the L1, L2
    factors of every layer over one optimizer buffer)."""
    out, off = [], 0
    for sh in shapes:
        n = 1
        for d in sh:
            n *= int(d)
        out.append(flat[off:off + n].view(*sh))
        off += n
    if off != flat.numel():
        raise ValueError("shapes do not cover the flat tensor")
    return out
