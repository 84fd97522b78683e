"""GPU parity with single-level constants (no double quantization): one fp32
absmax per block of 64, the scheme the walkthrough's double-quantization
section compares with (0.5 instead of 0.127 bit per parameter).  Dequant is
bit-exact against the oracle; the forward (every decode and tiled path) and
the backward meet the same tolerances as with double-quantized constants."""
import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import OTHER_CODEBOOKS, TOL_F32_W, TOL_SAME_W, Layer, bits

pytestmark = pytest.mark.gpu


def _oracle_w(layer):
    codes, absmax = nf4.quantize_blockwise(bits(layer.W_t), layer.codebook)
    cp = nf4.pack_codes(codes)
    wb = nf4.dequant_blocks(cp, absmax, layer.codebook)
    wf = nf4.dequant_blocks(cp, absmax, layer.codebook, out="f32")
    return (cp, absmax, wb, nf4.bf16_bits_to_f32(wb).reshape(layer.o, layer.h).astype(np.float64),
            wf.reshape(layer.o, layer.h).astype(np.float64))


@pytest.mark.parametrize("o,h", [(64, 192), (256, 512), (320, 1216), (1024, 4096)])
def test_single_level_dequant_bit_exact(o, h):
    layer = Layer(M=1, h=h, o=o, r=8, s=1.0, seed=o + h, outlier_frac=0.001)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook, double_quant=False)
    assert not Wq.double_quantized
    Wd = q.qlora_dequant(Wq)
    torch.cuda.synchronize()
    q.qlora_check_status()
    cp, absmax, wb, _, _ = _oracle_w(layer)
    assert np.array_equal(Wq.codes.cpu().numpy(), cp)
    assert np.array_equal(Wq.absmax.cpu().numpy().view(np.uint32), absmax.view(np.uint32))
    assert np.array_equal(bits(Wd), wb)


@pytest.mark.parametrize("M", [1, 2, 9, 16, 24, 300])
@pytest.mark.parametrize("h,o", [(512, 320), (1216, 1024)])
def test_single_level_forward_backward(M, h, o):
    layer = Layer(M=M, h=h, o=o, r=16, s=0.5, seed=7 * M + h)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook, double_quant=False)
    X, dY, L1, L2 = layer.X.cuda(), layer.dY.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y, T = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s)
    dX, dL1, dL2 = q.qlora_linear_bwd(Wq, X, dY, L1, L2, layer.s, T_saved=T)
    torch.cuda.synchronize()
    q.qlora_check_status()
    _, _, _, Wb, Wf = _oracle_w(layer)
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    Xo, dYo, L1o, L2o = (layer.f64(t) for t in (layer.X, layer.dY, layer.L1, layer.L2))
    rY, rT = nf4.lora_forward(Xo, Wb, L1o, L2o, layer.s)
    rdX, rdL1, rdL2, _, _ = nf4.lora_backward(Xo, dYo, Wb, L1o, L2o, layer.s)
    assert nf4.rel_max_err(f(Y), rY) <= TOL_SAME_W
    assert nf4.rel_max_err(f(T), rT) <= 1e-5
    assert nf4.rel_max_err(f(dX), rdX) <= TOL_SAME_W
    assert nf4.rel_max_err(f(dL1), rdL1) <= TOL_SAME_W
    assert nf4.rel_max_err(f(dL2), rdL2) <= TOL_SAME_W
    fY, _ = nf4.lora_forward(Xo, Wf, L1o, L2o, layer.s)
    assert nf4.rel_max_err(f(Y), fY) <= TOL_F32_W


@pytest.mark.parametrize("cb", list(OTHER_CODEBOOKS))
def test_single_level_other_codebooks(cb):
    layer = Layer(M=4, h=1024, o=640, r=16, s=0.5, seed=5, codebook=OTHER_CODEBOOKS[cb])
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook, double_quant=False)
    Y, _ = q.qlora_linear_fwd(Wq, layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda(), layer.s)
    torch.cuda.synchronize()
    _, _, _, Wb, _ = _oracle_w(layer)
    rY, _ = nf4.lora_forward(layer.f64(layer.X), Wb, layer.f64(layer.L1), layer.f64(layer.L2), layer.s)
    assert nf4.rel_max_err(Y.cpu().numpy().astype(np.float64), rY) <= TOL_SAME_W
