"""Binding checks that need no GPU: the Python entry points reject operands
whose shape, dtype or layout does not match the weight before any pointer
reaches the C ABI (which sees only pointers and could not tell an undersized
output from a correct one), and launch nothing when they do."""
import pytest
import torch

import bit_nf4_quantized_blockwise_b200 as q
from bit_nf4_quantized_blockwise_b200._lib import NF4Weight

O, H, M, R = 256, 512, 16, 8


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_blockwise_b200 import build
    build.build()
    return q.lib()


def _weight(o=O, h=H):
    n = o * h
    return NF4Weight(torch.zeros(n // 2, dtype=torch.uint8), torch.zeros(n // 64, dtype=torch.uint8),
                     torch.zeros(n // 16384, dtype=torch.float32), torch.zeros(1, dtype=torch.float32), o, h,
                     tuple(float(v) for v in range(-7, 9)))


def _operands(M=M):
    bf = torch.bfloat16
    return (torch.zeros(M, H, dtype=bf), torch.zeros(H, R, dtype=bf), torch.zeros(R, O, dtype=bf))


def _raises(fn, *args, match, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*args, **kw)


def test_forward_rejects_mismatched_outputs_before_any_launch(lib):
    Wq = _weight()
    X, L1, L2 = _operands()
    n0 = q.qlora_launch_count()
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, Y=torch.zeros(M, O - 64), match="Y has shape")
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, Y=torch.zeros(M - 1, O), match="Y has shape")
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, Y=torch.zeros(M, O, dtype=torch.float16), match="Y has dtype")
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, T_save=torch.zeros(M, R - 1), match="T has shape")
    _raises(q.qlora_linear_fwd, Wq, X[:, :H - 64], L1, L2, 1.0, match="X has shape")
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2[:, :O - 64], 1.0, match="L2 has shape")
    _raises(q.qlora_linear_fwd, Wq, X.float(), L1, L2, 1.0, match="X has dtype")
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, Y=torch.zeros(O, M).t(), match="Y must be contiguous")
    _raises(q.qlora_linear_fwd_noalloc, Wq, X, L1, L2, 1.0, Y=torch.zeros(M, O + 64), match="Y has shape")
    # well-formed host tensors pass the shape checks and stop at the device check
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, Y=torch.zeros(M, O), match="CUDA tensors")
    assert q.qlora_launch_count() == n0


def test_backward_rejects_mismatched_gradients_before_any_launch(lib):
    Wq = _weight()
    X, L1, L2 = _operands()
    dY = torch.zeros(M, O, dtype=torch.bfloat16)
    n0 = q.qlora_launch_count()
    _raises(q.qlora_linear_bwd, Wq, X, dY, L1, L2, 1.0, dX=torch.zeros(M, H - 64), match="dX has shape")
    _raises(q.qlora_linear_bwd, Wq, X, dY, L1, L2, 1.0, dL1=torch.zeros(H, R + 8), match="dL1 has shape")
    _raises(q.qlora_linear_bwd, Wq, X, dY, L1, L2, 1.0, dL2=torch.zeros(R, O - 64), match="dL2 has shape")
    _raises(q.qlora_linear_bwd, Wq, X, dY[:, :O - 64], L1, L2, 1.0, match="dY has shape")
    _raises(q.qlora_linear_bwd, Wq, X, dY, L1, L2, 1.0, T_saved=torch.zeros(M + 1, R), match="T has shape")
    _raises(q.qlora_linear_bwd, Wq, X, dY, L1, L2, 1.0, match="CUDA tensors")
    assert q.qlora_launch_count() == n0


def test_weight_arrays_must_match_its_shape(lib):
    X, L1, L2 = _operands()
    Wq = _weight()
    Wq.absmax_fp8 = Wq.absmax_fp8[:-1]
    _raises(q.qlora_linear_fwd, Wq, X, L1, L2, 1.0, match="absmax_fp8 must be")
    Wq = _weight()
    Wq.dq_scale = Wq.dq_scale.double()
    _raises(q.qlora_dequant, Wq, match="dq_scale must be")
    _raises(q.qlora_dequant, _weight(), out=torch.zeros(O, H + 64, dtype=torch.bfloat16), match="out has shape")
