"""GPU parity at the full benchmark sizes, in the launch configuration bench.py
times: LLaMA-7B-shaped linears at 4096 tokens and the three shapes of the
13B-shaped layer stack at 8192 tokens (fwd + bwd), the 65B-shaped
decode shapes (M = 1, 4, 16), and bulk quantize / dequant of one 65B-shaped
decoder layer's seven weights with 0.1% outliers.

Bit-exact items are compared on full tensors where the oracle is cheap
(absmax, FP8 constants, group scales, mean) and on seeded samples of blocks
otherwise; floating-point outputs on seeded row samples (rows of Y and dX
depend only on the same rows of X and dY) and in full for dL1 / dL2."""
import numpy as np
import pytest
import torch

import synth
from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import TOL_F32_W, TOL_SAME_W, bits

pytestmark = pytest.mark.gpu

CB = nf4.nf4_codebook()


def _oracle_absmax_full(wbits, block=64):
    out = np.empty(wbits.size // block, np.float32)
    step = 1 << 24
    for s in range(0, wbits.size, step):
        e = min(wbits.size, s + step)
        out[s // block:e // block] = nf4.block_absmax(wbits[s:e], block)
    return out


def _check_quantized(Wq, wbits, sample_blocks, rng):
    """Bit-exact check of a GPU-quantized weight against the oracle."""
    absmax = _oracle_absmax_full(wbits)
    e, sc, mu = nf4.double_quant(absmax)
    assert Wq.dq_mean.cpu().numpy().view(np.uint32)[0] == np.float32(mu).view(np.uint32)
    assert np.array_equal(Wq.dq_scale.cpu().numpy().view(np.uint32), sc.view(np.uint32))
    assert np.array_equal(Wq.absmax_fp8.cpu().numpy(), e)
    nb = absmax.size
    blocks = np.unique(np.concatenate([rng.integers(0, nb, sample_blocks), [0, nb - 1]]))
    idx = (blocks[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
    codes, am = nf4.quantize_blockwise(wbits[idx], CB)
    assert np.array_equal(am, absmax[blocks])
    gpu_codes = Wq.codes.cpu().numpy().reshape(-1, 32)[blocks].reshape(-1)
    assert np.array_equal(gpu_codes, nf4.pack_codes(codes))
    return absmax, e, sc, mu, blocks, nf4.pack_codes(codes)


def _oracle_weights(wbits, o, h):
    """The bf16 dequantized weight W' and the fp32 product q * c' it rounds."""
    codes, absmax = nf4.quantize_blockwise(wbits, CB)
    e, sc, mu = nf4.double_quant(absmax)
    cp = nf4.pack_codes(codes)
    wb = nf4.dequant(cp, e, sc, mu, CB)
    wf = nf4.dequant(cp, e, sc, mu, CB, out="f32")
    return (nf4.bf16_bits_to_f32(wb).reshape(o, h).astype(np.float64),
            wf.reshape(o, h).astype(np.float64))


def _oracle_wprime(wbits, o, h):
    return _oracle_weights(wbits, o, h)[0]


@pytest.mark.parametrize("h,o", [(4096, 4096), (4096, 11008), (11008, 4096)])
def test_llama7b_linear_fwd_bwd_full_size(h, o):
    _linear_fwd_bwd_full_size(4096, h, o, seed=1)


@pytest.mark.parametrize("h,o", [(5120, 5120), (5120, 13824), (13824, 5120)])
def test_llama13b_stack_linear_fwd_bwd_full_size(h, o):
    # the three shapes of the 13B-shaped layer stack (q/k/v/o, gate/up, down) at M = 8192
    _linear_fwd_bwd_full_size(8192, h, o, seed=5)


def _linear_fwd_bwd_full_size(M, h, o, seed):
    r, s = 64, 0.25
    rng = np.random.default_rng(h + o + M)
    W_t = synth.weight_t(o, h, seed=seed, tag=f"W{h}x{o}")
    X = synth.activations(M, h, seed=seed, tag=f"X{h}")
    dY = synth.activations(M, o, seed=seed, tag=f"dY{o}")
    L1, L2 = synth.lora_factors(h, r, o, seed=seed)
    Wq = q.quantize_weight(W_t.cuda(), CB)
    Y, T = q.qlora_linear_fwd(Wq, X.cuda(), L1.cuda(), L2.cuda(), s)
    dX, dL1, dL2 = q.qlora_linear_bwd(Wq, X.cuda(), dY.cuda(), L1.cuda(), L2.cuda(), s, T_saved=T)
    torch.cuda.synchronize()
    q.qlora_check_status()
    wbits = bits(W_t)
    _check_quantized(Wq, wbits, 4096, rng)
    Wb = _oracle_wprime(wbits, o, h)
    Xf, dYf = X.double().numpy(), dY.double().numpy()
    L1f, L2f = L1.double().numpy(), L2.double().numpy()
    rows = np.sort(rng.choice(M, 96, replace=False))
    rY, _ = nf4.lora_forward(Xf[rows], Wb, L1f, L2f, s)
    rdX, _, _, _, _ = nf4.lora_backward(Xf[rows], dYf[rows], Wb, L1f, L2f, s)
    assert nf4.rel_max_err(Y.cpu().numpy()[rows], rY) <= TOL_SAME_W
    assert nf4.rel_max_err(dX.cpu().numpy()[rows], rdX) <= TOL_SAME_W
    # dL1 = s X^T U and dL2 = s T^T dY in full (they do not involve W')
    T64 = Xf @ L1f
    U64 = dYf @ L2f.T
    assert nf4.rel_max_err(T.cpu().numpy(), T64) <= 1e-5
    assert nf4.rel_max_err(dL1.cpu().numpy(), s * (Xf.T @ U64)) <= TOL_SAME_W
    assert nf4.rel_max_err(dL2.cpu().numpy(), s * (T64.T @ dYf)) <= TOL_SAME_W


@pytest.mark.parametrize("h,o", [(8192, 8192), (8192, 22016)])
def test_65b_decode_shapes_full_size(h, o):
    r, s = 64, 0.25
    W_t = synth.weight_t(o, h, seed=2, tag=f"W{h}x{o}")
    L1, L2 = synth.lora_factors(h, r, o, seed=2)
    Wq = q.quantize_weight(W_t.cuda(), CB)
    Wb, Wf = _oracle_weights(bits(W_t), o, h)
    for M in (1, 4, 16):
        X = synth.activations(M, h, seed=M, tag="Xdec")
        Y, _ = q.qlora_linear_fwd(Wq, X.cuda(), L1.cuda(), L2.cuda(), s)
        torch.cuda.synchronize()
        q.qlora_check_status()
        args = (X.double().numpy(), L1.double().numpy(), L2.double().numpy())
        rY, _ = nf4.lora_forward(args[0], Wb, args[1], args[2], s)
        fY, _ = nf4.lora_forward(args[0], Wf, args[1], args[2], s)
        assert nf4.rel_max_err(Y.cpu().numpy(), rY) <= TOL_SAME_W, M
        assert nf4.rel_max_err(Y.cpu().numpy(), fY) <= TOL_F32_W, M


def test_65b_layer_bulk_quantize_dequant_full_size():
    d, ffn = 8192, 22016
    shapes = [(d, d)] * 4 + [(ffn, d), (ffn, d), (d, ffn)]   # q k v o, gate up (W^T [o][h]), down
    rng = np.random.default_rng(4)
    for i, (o, h) in enumerate(shapes):
        W_t = synth.weight_t(o, h, seed=4, tag=f"L65_{i}", outlier_frac=0.001)
        Wq = q.quantize_weight(W_t.cuda(), CB)
        Wd = q.qlora_dequant(Wq)
        torch.cuda.synchronize()
        q.qlora_check_status()
        wbits = bits(W_t)
        absmax, e, sc, mu, blocks, ocodes = _check_quantized(Wq, wbits, 2048, rng)
        cp = nf4.dequant_constants(e, sc, mu)[blocks]
        ref = nf4.dequant_blocks(ocodes, cp, CB).reshape(-1, 64)
        got = Wd.view(torch.int16).cpu().numpy().reshape(-1, 64)[blocks].view(np.uint16)
        assert np.array_equal(got, ref), i
        del W_t, Wq, Wd
        torch.cuda.empty_cache()
