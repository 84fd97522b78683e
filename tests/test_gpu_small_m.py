"""GPU parity of the small-M (decode) forward path, M <= 32 tokens, against the
CPU oracle; the same tolerances as the large-M path."""
import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import TOL_BF16_OUT, TOL_F32_W, TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu


def _fwd(layer, y_dtype=torch.float32):
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    Y, T = q.qlora_linear_fwd(Wq, layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda(), layer.s, y_dtype=y_dtype)
    torch.cuda.synchronize()
    q.qlora_check_status()
    return Y.float().cpu().numpy().astype(np.float64), T.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 31, 32])
@pytest.mark.parametrize("h,o", [(256, 256), (512, 320), (1024, 1088), (2048, 512), (320, 256), (1216, 1024)])
def test_small_m_forward(M, h, o):
    layer = Layer(M=M, h=h, o=o, r=64, s=0.25, seed=M * 31 + h + o)
    Y, T = _fwd(layer)
    Wb, Wf = layer.oracle_weights()
    X, L1, L2 = (layer.f64(t) for t in (layer.X, layer.L1, layer.L2))
    rY, rT = nf4.lora_forward(X, Wb, L1, L2, layer.s)
    fY, _ = nf4.lora_forward(X, Wf, L1, L2, layer.s)
    assert nf4.rel_max_err(T, rT) <= 1e-5
    # every path multiplies with the bf16 dequantized weight W'
    assert nf4.rel_max_err(Y, rY) <= TOL_SAME_W, nf4.rel_max_err(Y, rY)
    assert nf4.rel_max_err(Y, fY) <= TOL_F32_W


@pytest.mark.parametrize("M,r", [(4, 8), (4, 72), (4, 256), (1, 256), (12, 256), (16, 256), (2, 8)])
def test_small_m_ranks_and_bf16_output(M, r):
    layer = Layer(M=M, h=512, o=768, r=r, s=16.0 / r, seed=r + M)
    Y, _ = _fwd(layer, torch.bfloat16)
    X, L1, L2 = (layer.f64(t) for t in (layer.X, layer.L1, layer.L2))
    Wb, Wf = layer.oracle_weights()
    rY, _ = nf4.lora_forward(X, Wb, L1, L2, layer.s)
    assert nf4.rel_max_err(Y, rY) <= TOL_BF16_OUT


def test_small_and_large_paths_agree():
    # 32 tokens take the decode path, 33 the tiled path; the first 32 rows match.
    layer = Layer(M=33, h=1024, o=512, r=16, s=1.0, seed=77)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, L1, L2 = layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y33, _ = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s)
    Y32, _ = q.qlora_linear_fwd(Wq, X[:32].contiguous(), L1, L2, layer.s)
    torch.cuda.synchronize()
    a, b = Y32.cpu().numpy().astype(np.float64), Y33[:32].cpu().numpy().astype(np.float64)
    assert nf4.rel_max_err(a, b) <= 1e-5


def test_decode_kernels_agree_across_token_counts():
    # 8 tokens use one 8-column MMA group, 9..16 two, 17..32 the tcgen05 decode
    # kernel: the rows they share agree to fp32 summation-order noise.
    layer = Layer(M=17, h=2048, o=640, r=64, s=0.25, seed=91)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, L1, L2 = layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y = {}
    for M in (1, 8, 9, 16, 17):
        Y[M], _ = q.qlora_linear_fwd(Wq, X[:M].contiguous(), L1, L2, layer.s)
    torch.cuda.synchronize()
    q.qlora_check_status()
    f = {M: v.cpu().numpy().astype(np.float64) for M, v in Y.items()}
    for a, b in ((1, 8), (8, 9), (9, 16), (16, 17)):
        assert nf4.rel_max_err(f[a], f[b][:a]) <= 1e-5, (a, b)
