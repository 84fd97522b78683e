"""GPU parity of LoRA dropout on the adapter input (walkthrough "训练与推理
流程": 0.1 for 7B/13B, 0.05 for 33B/65B).  The keep mask is bit-exact against
the oracle's Philox4x32-10 draws on every path that applies it (the decode
rank-r kernel and the large-M masking kernel), and the forward and backward
meet the layer's tolerances against the oracle fed the identical bf16 W' and
the identical mask."""
import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import TOL_BF16_OUT, TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu


def _f(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M", [5, 20, 48, 300])
def test_dropout_mask_bit_exact(M):
    # with L1 = I (h = r) the product T = c (X * K) L1 exposes the mask element
    # by element: T[m][k] = fp32(c x[m][k]) where kept, 0 where dropped
    h = r = 256
    p, seed = 0.1, 0xDEADBEEF12345 + M
    layer = Layer(M=M, h=h, o=256, r=r, s=1.0, seed=M)
    X = torch.where(layer.X == 0, torch.ones_like(layer.X), layer.X)
    L1 = torch.eye(h, dtype=torch.bfloat16)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    _, T = q.qlora_linear_fwd(Wq, X.cuda(), L1.cuda(), layer.L2.cuda(), 1.0, dropout=p, seed=seed)
    torch.cuda.synchronize()
    q.qlora_check_status()
    keep = nf4.dropout_keep(M, h, p, seed)
    sc = nf4.dropout_scale(p)
    ref = np.where(keep, (X.float().numpy() * sc).astype(np.float32), np.float32(0))
    assert np.array_equal(T.cpu().numpy(), ref)
    assert 0.85 < keep.mean() < 0.95


@pytest.mark.parametrize("M", [1, 16, 24, 300])
@pytest.mark.parametrize("p", [0.1, 0.05])
def test_dropout_forward_backward(M, p):
    layer = Layer(M=M, h=512, o=640, r=64, s=0.25, seed=3 * M)
    seed = 77 + M
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, dY, L1, L2 = layer.X.cuda(), layer.dY.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y, T = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s, dropout=p, seed=seed)
    dX, dL1, dL2 = q.qlora_linear_bwd(Wq, X, dY, L1, L2, layer.s, T_saved=T, dropout=p, seed=seed)
    dX2, dL12, _ = q.qlora_linear_bwd(Wq, X, dY, L1, L2, layer.s, T_saved=None, dropout=p, seed=seed,
                                      dx_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    q.qlora_check_status()
    Wb, _ = layer.oracle_weights()
    keep = nf4.dropout_keep(M, layer.h, p, seed)
    sc = nf4.dropout_scale(p)
    args = [layer.f64(t) for t in (layer.X, layer.dY, layer.L1, layer.L2)]
    rY, rT = nf4.lora_forward_dropout(args[0], Wb, args[2], args[3], layer.s, keep, sc)
    rdX, rdL1, rdL2, _, _ = nf4.lora_backward_dropout(args[0], args[1], Wb, args[2], args[3], layer.s, keep, sc)
    assert nf4.rel_max_err(_f(T), rT) <= 1e-5
    assert nf4.rel_max_err(_f(Y), rY) <= TOL_SAME_W
    assert nf4.rel_max_err(_f(dX), rdX) <= TOL_SAME_W
    assert nf4.rel_max_err(_f(dL1), rdL1) <= TOL_SAME_W
    assert nf4.rel_max_err(_f(dL2), rdL2) <= TOL_SAME_W
    # recomputed T and a bf16 dX give the same gradients
    assert nf4.rel_max_err(_f(dX2), rdX) <= TOL_BF16_OUT
    assert nf4.rel_max_err(_f(dL12), rdL1) <= TOL_SAME_W
    # the dropped inputs receive only the base gradient dY W'^T
    base = args[1] @ Wb
    assert nf4.rel_max_err(_f(dX)[~keep], base[~keep]) <= TOL_SAME_W


def test_zero_rate_matches_the_plain_calls():
    layer = Layer(M=200, h=512, o=512, r=16, s=0.5, seed=2)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, dY, L1, L2 = layer.X.cuda(), layer.dY.cuda(), layer.L1.cuda(), layer.L2.cuda()
    L = q.lib()
    # the C entry point with p = 0
    import ctypes
    P = ctypes.c_void_p
    Y0 = torch.empty(200, 512, device="cuda")
    ws = torch.empty(L.qlora_linear_fwd_dropout_workspace_size(512, 512, 200, 16), dtype=torch.uint8, device="cuda")
    st = Wq.struct()
    rc = L.qlora_linear_fwd_dropout(ctypes.byref(st), P(X.data_ptr()), 200, P(L1.data_ptr()), P(L2.data_ptr()), 16,
                                    0.5, 0.0, 5, P(Y0.data_ptr()), 0, None, P(ws.data_ptr()), ws.numel(),
                                    P(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    assert L.qlora_linear_fwd_dropout(ctypes.byref(st), P(X.data_ptr()), 200, P(L1.data_ptr()), P(L2.data_ptr()),
                                      16, 0.5, 1.0, 5, P(Y0.data_ptr()), 0, None, P(ws.data_ptr()), ws.numel(),
                                      None) == 4  # p = 1 is rejected
    Y1, _ = q.qlora_linear_fwd(Wq, X, L1, L2, 0.5)
    torch.cuda.synchronize()
    assert nf4.rel_max_err(_f(Y0), _f(Y1)) <= 1e-6
