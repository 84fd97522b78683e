"""GPU parity of the adapter merge into the bf16 dequantized base,
W_m = bf16(W' + s L1 L2) (QLoRA glossary, pitfalls entry), against the
oracle's fp64 sum rounded once.  The kernel forms s L1 L2 in fp32 on the
tensor cores before its single bf16 rounding, so an element may land on the
other bf16 neighbour only where the exact value sits within fp32 noise of a
bf16 midpoint: every element is within one bf16 step of the oracle and
almost all are identical.  Without an adapter the merge is the dequantized
weight bit for bit."""
import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import Layer, bits

pytestmark = pytest.mark.gpu


def _key(b):
    """bf16 bit patterns -> integers in value order (one step = one bf16 ulp)."""
    b = b.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _check(layer, double_quant=True, min_exact=0.999):
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook, double_quant=double_quant)
    Wd = q.qlora_dequant(Wq)
    Wm = q.qlora_merge_bf16(Wq, layer.L1.cuda(), layer.L2.cuda(), layer.s)
    torch.cuda.synchronize()
    q.qlora_check_status()
    wd = bits(Wd).reshape(layer.o, layer.h)
    L1, L2 = layer.f64(layer.L1), layer.f64(layer.L2)
    ref = nf4.merge_adapter(wd, L1, L2, layer.s)
    got = bits(Wm).reshape(layer.o, layer.h)
    # exact value, and the size of what was summed (fp32 noise is relative to it)
    wp = nf4.bf16_bits_to_f32(wd).astype(np.float64)
    exact = wp + layer.s * (L1 @ L2).T
    mag = np.abs(wp) + abs(layer.s) * (np.abs(L1) @ np.abs(L2)).T
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    err = np.abs(nf4.bf16_bits_to_f32(got).astype(np.float64) - exact)
    # within one bf16 step of the exact value, beyond it only by fp32 noise
    # (where W' and s L1 L2 nearly cancel)
    assert np.all(err <= ulp + 2.0 ** -20 * mag)
    steps = np.abs(_key(got) - _key(ref))
    assert np.mean(steps == 0) >= min_exact, np.mean(steps == 0)
    assert np.mean(steps <= 1) >= 0.99999
    return Wq, Wd


@pytest.mark.parametrize("o,h,r", [(256, 256, 8), (512, 1216, 72), (1024, 4096, 64), (4096, 4096, 64),
                                   (576, 512, 256)])
def test_merge_matches_oracle(o, h, r):
    _check(Layer(M=1, h=h, o=o, r=r, s=16.0 / r, seed=o + h + r))


def test_merge_single_level_constants():
    _check(Layer(M=1, h=1024, o=640, r=64, s=0.25, seed=9), double_quant=False)


def test_merge_without_adapter_is_the_dequantized_weight():
    layer = Layer(M=1, h=512, o=384, r=16, s=2.0, seed=10)
    layer.L2 = torch.zeros_like(layer.L2)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    Wd = q.qlora_dequant(Wq)
    Wm = q.qlora_merge_bf16(Wq, layer.L1.cuda(), layer.L2.cuda(), layer.s)
    torch.cuda.synchronize()
    assert np.array_equal(bits(Wm), bits(Wd))


def test_merged_weight_reproduces_the_adapter_forward():
    layer = Layer(M=64, h=1024, o=512, r=64, s=0.25, seed=11)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    Y, _ = q.qlora_linear_fwd(Wq, layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda(), layer.s)
    Wm = q.qlora_merge_bf16(Wq, layer.L1.cuda(), layer.L2.cuda(), layer.s)
    torch.cuda.synchronize()
    Ym = layer.f64(layer.X) @ nf4.bf16_bits_to_f32(bits(Wm)).reshape(layer.o, layer.h).astype(np.float64).T
    assert nf4.rel_max_err(Ym, Y.cpu().numpy().astype(np.float64)) <= 2.0 ** -8
