"""GPU parity of the QLoRA linear layer (forward and backward) against the
CPU oracle, at sizes the oracle finishes in seconds that still span several
tiles and ragged tails."""
import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import OTHER_CODEBOOKS, TOL_BF16_OUT, TOL_F32_W, TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu


def _run(layer: Layer, y_dtype=torch.float32, use_saved_T=True, min_workspace=False):
    cb = layer.codebook
    Wq = q.quantize_weight(layer.W_t.cuda(), cb)
    X, dY = layer.X.cuda(), layer.dY.cuda()
    L1, L2 = layer.L1.cuda(), layer.L2.cuda()
    wsf = wsb = None
    if min_workspace:
        # the smallest accepted workspaces: W' is never materialised
        L = q.lib()
        args = (layer.o, layer.h, layer.M, layer.r)
        wsf = torch.empty(L.qlora_linear_fwd_workspace_min_size(*args), dtype=torch.uint8, device="cuda")
        wsb = torch.empty(L.qlora_linear_bwd_workspace_min_size(*args), dtype=torch.uint8, device="cuda")
    Y, T = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s, y_dtype=y_dtype, ws=wsf)
    dX, dL1, dL2 = q.qlora_linear_bwd(Wq, X, dY, L1, L2, layer.s, T_saved=T if use_saved_T else None,
                                      dx_dtype=y_dtype, ws=wsb)
    torch.cuda.synchronize()
    q.qlora_check_status()
    return [t.float().cpu().numpy().astype(np.float64) for t in (Y, T, dX, dL1, dL2)]


def _check(layer: Layer, y_dtype=torch.float32, use_saved_T=True, min_workspace=False):
    Y, T, dX, dL1, dL2 = _run(layer, y_dtype, use_saved_T, min_workspace)
    Wb, Wf = layer.oracle_weights()
    X, dY, L1, L2 = (layer.f64(t) for t in (layer.X, layer.dY, layer.L1, layer.L2))
    rY, rT = nf4.lora_forward(X, Wb, L1, L2, layer.s)
    rdX, rdL1, rdL2, _, _ = nf4.lora_backward(X, dY, Wb, L1, L2, layer.s)
    tol = TOL_SAME_W if y_dtype == torch.float32 else TOL_BF16_OUT
    errs = {"Y": nf4.rel_max_err(Y, rY), "dX": nf4.rel_max_err(dX, rdX)}
    assert errs["Y"] <= tol and errs["dX"] <= tol, errs
    assert nf4.rel_max_err(T, rT) <= 1e-5
    assert nf4.rel_max_err(dL1, rdL1) <= TOL_SAME_W, nf4.rel_max_err(dL1, rdL1)
    assert nf4.rel_max_err(dL2, rdL2) <= TOL_SAME_W, nf4.rel_max_err(dL2, rdL2)
    fY, _ = nf4.lora_forward(X, Wf, L1, L2, layer.s)
    fdX, _, _, _, _ = nf4.lora_backward(X, dY, Wf, L1, L2, layer.s)
    assert nf4.rel_max_err(Y, fY) <= TOL_F32_W and nf4.rel_max_err(dX, fdX) <= TOL_F32_W
    return errs


def test_small_layer_config():
    # W 256x256 N(0, 0.02), X 16x256, r = 8, s = 2, seed 0.
    _check(Layer(M=16, h=256, o=256, r=8, s=2.0, seed=0))


@pytest.mark.parametrize("M", [1, 17, 129, 256, 300, 513])
def test_ragged_tokens(M):
    _check(Layer(M=M, h=512, o=512, r=16, s=0.5, seed=M))


@pytest.mark.parametrize("h,o", [(256, 576), (576, 256), (1024, 320), (320, 1024)])
def test_ragged_feature_tiles(h, o):
    _check(Layer(M=200, h=h, o=o, r=64, s=0.25, seed=h + o))


@pytest.mark.parametrize("r", [8, 24, 64, 72, 128, 256])
def test_ranks(r):
    _check(Layer(M=160, h=512, o=256, r=r, s=16.0 / r, seed=r))


def test_bf16_outputs_and_recomputed_T():
    _check(Layer(M=300, h=512, o=768, r=64, s=0.25, seed=5), y_dtype=torch.bfloat16, use_saved_T=False)


def test_zero_adapter_gives_plain_product():
    layer = Layer(M=64, h=256, o=256, r=8, s=2.0, seed=6)
    layer.L2 = torch.zeros_like(layer.L2)
    Y, T, dX, dL1, dL2 = _run(layer)
    Wb, _ = layer.oracle_weights()
    X, dY = layer.f64(layer.X), layer.f64(layer.dY)
    assert nf4.rel_max_err(Y, X @ Wb.T) <= TOL_SAME_W
    assert not np.any(dL1)


def test_deep_reduction_and_many_tiles():
    # several 256x256 output tiles in both directions, long K on both passes
    _check(Layer(M=512, h=2048, o=1536, r=64, s=0.25, seed=11, outlier_frac=0.001))


@pytest.mark.parametrize("M,h,o,r", [(2048, 1024, 4096, 64), (2560, 2048, 576, 16), (2304, 320, 2304, 256)])
def test_many_tiles_odd_depths(M, h, o, r):
    # More 256 x 256 output tiles than SMs in one direction or the other (128
    # forward tiles; 80 backward tiles over an odd number of 64-deep stages),
    # and the deepest LoRA extension (r = 256) behind an odd number of stages.
    _check(Layer(M=M, h=h, o=o, r=r, s=16.0 / r, seed=M + h + o))


@pytest.mark.parametrize("min_workspace", [False, True])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_both_paths_at_many_tokens(min_workspace, y_dtype):
    # From 1024 tokens a full workspace selects W' dequantized once into it
    # plus the pair-tile bf16 GEMM; the minimum workspace keeps the fused
    # dequant-GEMM.  Both must meet the same bar, with a ragged token tail.
    _check(Layer(M=1280 + 40, h=576, o=768, r=64, s=0.25, seed=21), y_dtype=y_dtype, min_workspace=min_workspace)


@pytest.mark.parametrize("cb", list(OTHER_CODEBOOKS))
@pytest.mark.parametrize("M", [1, 16, 300])
def test_other_4bit_codebooks(cb, M):
    # Int4 and the FP4 variants run through the same kernels as NF4, the
    # codebook being data: the CUDA-core and tensor-core decode paths and the
    # tiled path, forward and backward.
    _check(Layer(M=M, h=1024, o=640, r=16, s=0.5, seed=M + 3, codebook=OTHER_CODEBOOKS[cb]))
