"""ctypes binding of libqlora.so.

Argument marshalling only: every computation runs in the CUDA library.  The
functions carry the C entry points' names and take torch tensors (device
memory and the current stream come from PyTorch).  There is no fallback: if
the library is missing or a call fails, they raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_OK = 0
QLORA_DTYPE_F32 = 0
QLORA_DTYPE_BF16 = 1

_c_void_p = ctypes.c_void_p
_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_size = ctypes.c_size_t
_c_float = ctypes.c_float


class qlora_adamw_t(ctypes.Structure):
    """Mirror of the C struct qlora_adamw_t."""
    _fields_ = [("lr", _c_float), ("beta1", _c_float), ("beta2", _c_float), ("eps", _c_float),
                ("weight_decay", _c_float), ("max_grad_norm", _c_float), ("step", ctypes.c_int32)]


class qlora_nf4_t(ctypes.Structure):
    """Mirror of the C struct qlora_nf4_t."""
    _fields_ = [
        ("codes", _c_void_p),
        ("absmax_fp8", _c_void_p),
        ("dq_scale", _c_void_p),
        ("dq_mean", _c_void_p),
        ("o", _c_i64),
        ("h", _c_i64),
        ("codebook", _c_float * 16),
        ("block", ctypes.c_int32),
        ("dq_block", ctypes.c_int32),
        ("absmax", _c_void_p),
    ]


EXPORTS = {
    "qlora_status_string": (ctypes.c_char_p, [_c_int]),
    "qlora_version": (_c_int, []),
    "qlora_quantize_nf4": (_c_int, [_c_void_p, _c_i64, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "qlora_double_quant_workspace_size": (_c_size, [_c_i64, _c_int]),
    "qlora_double_quant": (_c_int, [_c_void_p, _c_i64, _c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                    _c_size, _c_void_p]),
    "qlora_dequant": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_void_p]),
    "qlora_linear_fwd_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_fwd": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_i64, _c_void_p, _c_void_p, _c_int,
                                  _c_float, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_size, _c_void_p]),
    "qlora_linear_bwd_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_bwd": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_void_p, _c_i64, _c_void_p, _c_void_p,
                                  _c_int, _c_float, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p,
                                  _c_size, _c_void_p]),
    "qlora_linear_fwd_dropout_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_bwd_dropout_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_fwd_workspace_min_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_bwd_workspace_min_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_fwd_dropout_workspace_min_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_bwd_dropout_workspace_min_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_fwd_dropout": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_i64, _c_void_p, _c_void_p, _c_int,
                                          _c_float, _c_float, ctypes.c_uint64, _c_void_p, _c_int, _c_void_p,
                                          _c_void_p, _c_size, _c_void_p]),
    "qlora_linear_bwd_dropout": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_void_p, _c_i64, _c_void_p,
                                          _c_void_p, _c_int, _c_float, _c_float, ctypes.c_uint64, _c_void_p,
                                          _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p, _c_size, _c_void_p]),
    "qlora_paged_alloc": (_c_int, [_c_size, ctypes.POINTER(_c_void_p)]),
    "qlora_paged_free": (_c_int, [_c_void_p]),
    "qlora_paged_advise": (_c_int, [_c_void_p, _c_size, _c_int]),
    "qlora_paged_prefetch": (_c_int, [_c_void_p, _c_size, _c_int, _c_void_p]),
    "qlora_grad_sqnorm": (_c_int, [_c_void_p, _c_i64, _c_void_p, _c_void_p]),
    "qlora_adamw_step": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_i64, _c_void_p,
                                  _c_void_p, _c_void_p]),
    "qlora_check_status": (_c_int, [_c_void_p]),
    "qlora_debug_wait_tags": (ctypes.c_uint, []),
    "qlora_debug_wait_probe": (_c_int, [ctypes.c_uint64, _c_void_p]),
    "qlora_linear_fwd_noalloc": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_i64, _c_void_p, _c_void_p,
                                          _c_int, _c_float, _c_void_p, _c_int, _c_void_p, _c_void_p]),
    "qlora_nf4_boundaries": (_c_int, [_c_void_p, _c_void_p]),
    "qlora_merge_bf16": (_c_int, [ctypes.POINTER(qlora_nf4_t), _c_void_p, _c_void_p, _c_int, _c_float, _c_void_p,
                                  _c_void_p]),
    "qlora_nf4_codebook": (_c_int, [_c_void_p]),
    "qlora_launch_count": (_c_i64, []),
    "qlora_trace_enable": (None, [_c_int]),
    "qlora_trace_read": (_c_int, [_c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_c_i64)]),
    "qlora_kernel_family_name": (ctypes.c_char_p, [_c_int]),
}

KERNEL_FAMILIES = 11

_LIB = None


def lib() -> ctypes.CDLL:
    """Loads libqlora.so (built in-tree by build.py); raises if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_nf4_quantized_blockwise_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


class QLoRAError(RuntimeError):
    def __init__(self, what: str, status: int):
        self.status = status
        super().__init__(f"{what} failed: {lib().qlora_status_string(status).decode()} (status {status})")


def _check(status: int, what: str) -> None:
    if status != QLORA_OK:
        raise QLoRAError(what, status)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else _c_void_p(t.data_ptr())


def _stream(dev: torch.device) -> _c_void_p:
    return _c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _require_cuda(*ts: torch.Tensor) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libqlora takes CUDA tensors (device memory)")
        if not t.is_contiguous():
            raise ValueError("libqlora takes contiguous tensors")
        dev = t.device if dev is None else dev
    return dev


def _same_device(*ts: Optional[torch.Tensor]) -> None:
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"operands are on different devices: {sorted(str(d) for d in devs)}")


def _need(t: Optional[torch.Tensor], name: str, shape, dtypes) -> None:
    """Shape, dtype and layout of one operand (None = not passed)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {[str(d) for d in dtypes]}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_weight(Wq: "NF4Weight") -> None:
    """The weight's device arrays hold exactly the sizes (o, h) imply."""
    n = Wq.o * Wq.h
    arrays = [(Wq.codes, "codes", n // 2, torch.uint8)]
    if Wq.absmax is not None:
        arrays.append((Wq.absmax, "absmax", n // 64, torch.float32))
    else:
        arrays += [(Wq.absmax_fp8, "absmax_fp8", n // 64, torch.uint8),
                   (Wq.dq_scale, "dq_scale", max(n // (64 * 256), 1), torch.float32),
                   (Wq.dq_mean, "dq_mean", 1, torch.float32)]
    for t, name, numel, dt in arrays:
        if t is None:
            raise ValueError(f"{name} is missing")
        if t.numel() != numel or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dt} tensor of {numel} elements for o={Wq.o}, h={Wq.h}; "
                             f"got {t.dtype} with {t.numel()} elements")


def _check_linear(Wq: "NF4Weight", X, L1, L2, Y=None, T=None, dY=None, dX=None, dL1=None, dL2=None):
    """Checks every linear-layer operand against the weight's (o, h) and the
    token count M = X.shape[0] before any pointer reaches the library: the C
    ABI only sees pointers, so an undersized output would be written past its
    end on the device.  Returns (M, r)."""
    _check_weight(Wq)
    o, h = Wq.o, Wq.h
    if X.dim() != 2 or X.shape[1] != h:
        raise ValueError(f"X has shape {tuple(X.shape)}, expected (M, {h})")
    if L1.dim() != 2 or L1.shape[0] != h:
        raise ValueError(f"L1 has shape {tuple(L1.shape)}, expected ({h}, r)")
    M, r = X.shape[0], L1.shape[1]
    _need(X, "X", (M, h), (torch.bfloat16,))
    _need(L1, "L1", (h, r), (torch.bfloat16,))
    _need(L2, "L2", (r, o), (torch.bfloat16,))
    _need(Y, "Y", (M, o), (torch.float32, torch.bfloat16))
    _need(T, "T", (M, r), (torch.float32,))
    _need(dY, "dY", (M, o), (torch.bfloat16,))
    _need(dX, "dX", (M, h), (torch.float32, torch.bfloat16))
    _need(dL1, "dL1", (h, r), (torch.float32,))
    _need(dL2, "dL2", (r, o), (torch.float32,))
    _same_device(Wq.codes, Wq.absmax_fp8, Wq.dq_scale, Wq.dq_mean, Wq.absmax, X, L1, L2, Y, T, dY, dX, dL1, dL2)
    return M, r


def _codebook_array(codebook: Sequence[float]):
    vals = [float(v) for v in (codebook.tolist() if hasattr(codebook, "tolist") else codebook)]
    if len(vals) != 16:
        raise ValueError("codebook must have 16 entries")
    return (_c_float * 16)(*vals)


@dataclass
class NF4Weight:
    """A blockwise-quantized NF4 weight W^T[o][h] held in device memory:
    double-quantized constants (absmax_fp8, dq_scale, dq_mean), or, with
    ``absmax`` set, one fp32 constant per block of 64 (no double quantization;
    the other three are then None)."""
    codes: torch.Tensor                  # uint8 [o*h/2]
    absmax_fp8: Optional[torch.Tensor]   # uint8 [o*h/64]
    dq_scale: Optional[torch.Tensor]     # fp32  [o*h/64/256]
    dq_mean: Optional[torch.Tensor]      # fp32  [1]
    o: int
    h: int
    codebook: Tuple[float, ...]
    absmax: Optional[torch.Tensor] = None   # fp32 [o*h/64], single-level constants

    @property
    def double_quantized(self) -> bool:
        return self.absmax is None

    def struct(self) -> qlora_nf4_t:
        s = qlora_nf4_t()
        s.codes = self.codes.data_ptr()
        s.absmax_fp8 = self.absmax_fp8.data_ptr() if self.absmax_fp8 is not None else None
        s.dq_scale = self.dq_scale.data_ptr() if self.dq_scale is not None else None
        s.dq_mean = self.dq_mean.data_ptr() if self.dq_mean is not None else None
        s.o = self.o
        s.h = self.h
        s.codebook = _codebook_array(self.codebook)
        s.block = 64
        s.dq_block = 256
        s.absmax = self.absmax.data_ptr() if self.absmax is not None else None
        return s


# ---------------------------------------------------------------- entry points

def qlora_quantize_nf4(W: torch.Tensor, codebook: Sequence[float], block: int = 64,
                       codes: Optional[torch.Tensor] = None, absmax: Optional[torch.Tensor] = None):
    """Blockwise absmax NF4 quantization of a bf16 tensor.  Returns (codes, absmax)."""
    dev = _require_cuda(W)
    if W.dtype != torch.bfloat16:
        raise ValueError("W must be bf16")
    n = W.numel()
    if codes is None:
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    if absmax is None:
        absmax = torch.empty(max(n // 64, 1), dtype=torch.float32, device=dev)
    cb = _codebook_array(codebook)
    with torch.cuda.device(dev):
        _check(lib().qlora_quantize_nf4(_p(W), n, ctypes.cast(cb, _c_void_p), block, _p(codes), _p(absmax),
                                        _stream(dev)), "qlora_quantize_nf4")
    return codes, absmax


def qlora_double_quant(absmax: torch.Tensor, dq_block: int = 256, absmax_fp8=None, dq_scale=None,
                       dq_mean=None, ws=None):
    """Double quantization of fp32 block constants.  Returns (absmax_fp8, dq_scale, dq_mean)."""
    dev = _require_cuda(absmax)
    nb = absmax.numel()
    if absmax_fp8 is None:
        absmax_fp8 = torch.empty(nb, dtype=torch.uint8, device=dev)
    if dq_scale is None:
        dq_scale = torch.empty(max(nb // 256, 1), dtype=torch.float32, device=dev)
    if dq_mean is None:
        dq_mean = torch.empty(1, dtype=torch.float32, device=dev)
    L = lib()
    wsb = L.qlora_double_quant_workspace_size(nb, dq_block)
    if ws is None:
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(L.qlora_double_quant(_p(absmax), nb, dq_block, _p(absmax_fp8), _p(dq_scale), _p(dq_mean), _p(ws),
                                    ws.numel(), _stream(dev)), "qlora_double_quant")
    return absmax_fp8, dq_scale, dq_mean


def quantize_weight(W_t: torch.Tensor, codebook: Sequence[float], double_quant: bool = True) -> NF4Weight:
    """qlora_quantize_nf4 then qlora_double_quant of a bf16 W^T[o][h]; with
    double_quant=False the fp32 block constants are kept as they are."""
    o, h = W_t.shape
    codes, absmax = qlora_quantize_nf4(W_t, codebook)
    cb = tuple(float(v) for v in codebook)
    if not double_quant:
        return NF4Weight(codes, None, None, None, o, h, cb, absmax=absmax)
    fp8, sc, mu = qlora_double_quant(absmax)
    return NF4Weight(codes, fp8, sc, mu, o, h, cb)


def qlora_dequant(Wq: NF4Weight, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """doubleDequant of the whole weight to bf16 [o][h]."""
    _check_weight(Wq)
    _need(out, "out", (Wq.o, Wq.h), (torch.bfloat16,))
    dev = _require_cuda(Wq.codes, out)
    if out is None:
        out = torch.empty(Wq.o, Wq.h, dtype=torch.bfloat16, device=dev)
    s = Wq.struct()
    with torch.cuda.device(dev):
        _check(lib().qlora_dequant(ctypes.byref(s), _p(out), _stream(dev)), "qlora_dequant")
    return out


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return QLORA_DTYPE_F32
    if dt == torch.bfloat16:
        return QLORA_DTYPE_BF16
    raise ValueError("output dtype must be float32 or bfloat16")


def qlora_linear_fwd(Wq: NF4Weight, X: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, s: float,
                     y_dtype: torch.dtype = torch.float32, save_T: bool = True,
                     Y: Optional[torch.Tensor] = None, T_save: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, dropout: float = 0.0, seed: int = 0):
    """Y = X W' + s X L1 L2.  Returns (Y, T) with T = X L1 in fp32 (None unless save_T).
    With dropout > 0 the adapter input is X with LoRA dropout (rate `dropout`,
    Philox key `seed`; see qlora_linear_fwd_dropout) and T is its scaled product."""
    M, r = _check_linear(Wq, X, L1, L2, Y=Y, T=T_save)
    dev = _require_cuda(X, L1, L2, Y, T_save, Wq.codes)
    if Y is None:
        Y = torch.empty(M, Wq.o, dtype=y_dtype, device=dev)
    if T_save is None and save_T:
        T_save = torch.empty(M, r, dtype=torch.float32, device=dev)
    L = lib()
    drop = dropout != 0.0
    wsb = (L.qlora_linear_fwd_dropout_workspace_size if drop else L.qlora_linear_fwd_workspace_size)(Wq.o, Wq.h, M, r)
    if ws is None or ws.numel() * ws.element_size() < wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    st = Wq.struct()
    with torch.cuda.device(dev):
        if drop:
            _check(L.qlora_linear_fwd_dropout(ctypes.byref(st), _p(X), M, _p(L1), _p(L2), r, float(s), float(dropout),
                                              int(seed), _p(Y), _dtype_code(Y.dtype), _p(T_save), _p(ws),
                                              ws.numel() * ws.element_size(), _stream(dev)),
                   "qlora_linear_fwd_dropout")
        else:
            _check(L.qlora_linear_fwd(ctypes.byref(st), _p(X), M, _p(L1), _p(L2), r, float(s), _p(Y),
                                      _dtype_code(Y.dtype), _p(T_save), _p(ws), ws.numel() * ws.element_size(),
                                      _stream(dev)),
                   "qlora_linear_fwd")
    return Y, T_save


def qlora_linear_bwd(Wq: NF4Weight, X: torch.Tensor, dY: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor,
                     s: float, T_saved: Optional[torch.Tensor] = None, dx_dtype: torch.dtype = torch.float32,
                     dX: Optional[torch.Tensor] = None, dL1: Optional[torch.Tensor] = None,
                     dL2: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     dropout: float = 0.0, seed: int = 0):
    """Returns (dX, dL1, dL2) of <Y, dY>; W is frozen (no dW).  dropout / seed
    must be the forward's (LoRA dropout on the adapter input)."""
    M, r = _check_linear(Wq, X, L1, L2, T=T_saved, dY=dY, dX=dX, dL1=dL1, dL2=dL2)
    dev = _require_cuda(X, dY, L1, L2, T_saved, dX, dL1, dL2, Wq.codes)
    if dX is None:
        dX = torch.empty(M, Wq.h, dtype=dx_dtype, device=dev)
    if dL1 is None:
        dL1 = torch.empty(Wq.h, r, dtype=torch.float32, device=dev)
    if dL2 is None:
        dL2 = torch.empty(r, Wq.o, dtype=torch.float32, device=dev)
    L = lib()
    drop = dropout != 0.0
    wsb = (L.qlora_linear_bwd_dropout_workspace_size if drop else L.qlora_linear_bwd_workspace_size)(Wq.o, Wq.h, M, r)
    if ws is None or ws.numel() * ws.element_size() < wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    st = Wq.struct()
    nbytes = ws.numel() * ws.element_size()
    with torch.cuda.device(dev):
        if drop:
            _check(L.qlora_linear_bwd_dropout(ctypes.byref(st), _p(X), _p(dY), M, _p(L1), _p(L2), r, float(s),
                                              float(dropout), int(seed), _p(T_saved), _p(dX), _dtype_code(dX.dtype),
                                              _p(dL1), _p(dL2), _p(ws), nbytes, _stream(dev)),
                   "qlora_linear_bwd_dropout")
        else:
            _check(L.qlora_linear_bwd(ctypes.byref(st), _p(X), _p(dY), M, _p(L1), _p(L2), r, float(s), _p(T_saved),
                                      _p(dX), _dtype_code(dX.dtype), _p(dL1), _p(dL2), _p(ws), nbytes, _stream(dev)),
                   "qlora_linear_bwd")
    return dX, dL1, dL2


def qlora_linear_fwd_noalloc(Wq: NF4Weight, X: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, s: float,
                             Y: torch.Tensor, T_save: Optional[torch.Tensor] = None) -> None:
    """qlora_linear_fwd without a workspace, for callers that cannot allocate
    device memory: the library's built-in scratch array is used instead (see
    include/qlora.h for its size limit and sharing rules).  Y (and T_save) are
    caller-provided outputs; nothing is allocated."""
    _check_linear(Wq, X, L1, L2, Y=Y, T=T_save)
    dev = _require_cuda(X, L1, L2, Y, T_save, Wq.codes)
    st = Wq.struct()
    with torch.cuda.device(dev):
        _check(lib().qlora_linear_fwd_noalloc(ctypes.byref(st), _p(X), X.shape[0], _p(L1), _p(L2), L1.shape[1],
                                              float(s), _p(Y), _dtype_code(Y.dtype), _p(T_save), _stream(dev)),
               "qlora_linear_fwd_noalloc")


def qlora_merge_bf16(Wq: NF4Weight, L1: torch.Tensor, L2: torch.Tensor, s: float,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The adapter merged into the bf16 dequantized base: W_m^T = bf16(W'^T + s (L1 L2)^T), [o][h]."""
    _check_weight(Wq)
    o, h = Wq.o, Wq.h
    if L1.dim() != 2 or L1.shape[0] != h:
        raise ValueError(f"L1 has shape {tuple(L1.shape)}, expected ({h}, r)")
    r = L1.shape[1]
    _need(L1, "L1", (h, r), (torch.bfloat16,))
    _need(L2, "L2", (r, o), (torch.bfloat16,))
    _need(out, "out", (o, h), (torch.bfloat16,))
    _same_device(Wq.codes, L1, L2, out)
    dev = _require_cuda(Wq.codes, L1, L2, out)
    if out is None:
        out = torch.empty(o, h, dtype=torch.bfloat16, device=dev)
    st = Wq.struct()
    with torch.cuda.device(dev):
        _check(lib().qlora_merge_bf16(ctypes.byref(st), _p(L1), _p(L2), r, float(s), _p(out), _stream(dev)),
               "qlora_merge_bf16")
    return out


def qlora_check_status(device: Optional[torch.device] = None) -> None:
    """Waits for the current stream and raises if a kernel pipeline wait gave up."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib().qlora_check_status(_stream(dev)), "qlora_check_status")


def qlora_nf4_codebook() -> Tuple[float, ...]:
    """Host-only: the library's 16 NF4 code values (fp32, increasing)."""
    out = (_c_float * 16)()
    _check(lib().qlora_nf4_codebook(ctypes.cast(out, _c_void_p)), "qlora_nf4_codebook")
    return tuple(float(v) for v in out)


def qlora_nf4_boundaries(codebook: Sequence[float]):
    """Host-only: the quantizer's per-significand decision table, uint16 [128][16]."""
    import numpy as np
    out = np.zeros((128, 16), dtype=np.uint16)
    cb = _codebook_array(codebook)
    _check(lib().qlora_nf4_boundaries(ctypes.cast(cb, _c_void_p), out.ctypes.data_as(_c_void_p)),
           "qlora_nf4_boundaries")
    return out


def qlora_launch_count() -> int:
    """Number of kernels this library has launched in this process."""
    return int(lib().qlora_launch_count())


def qlora_trace_enable(on: bool) -> None:
    lib().qlora_trace_enable(1 if on else 0)


def qlora_trace_read() -> dict:
    """{family name: (total device ms, launches)} of the traced launches; clears them."""
    out = {}
    L = lib()
    for f in range(KERNEL_FAMILIES):
        ms = ctypes.c_double()
        n = _c_i64()
        _check(L.qlora_trace_read(f, ctypes.byref(ms), ctypes.byref(n)), "qlora_trace_read")
        out[L.qlora_kernel_family_name(f).decode()] = (ms.value, int(n.value))
    return out
