"""Shared helpers of the GPU parity tests: seeded inputs from ``synth``, the
oracle's expected values, and the tolerances the tests apply."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import nf4

# Tolerances (max|out - ref| / max|ref| per tensor), stated for this layer:
#  - against the fp64 oracle fed the identical bf16 dequantized weight;
TOL_SAME_W = 1e-3
#  - against the oracle whose weight keeps the fp32 product q * c' unrounded;
TOL_F32_W = 2e-2
#  - bf16 outputs: one bf16 rounding (2^-8 relative to the largest entry) on top.
TOL_BF16_OUT = 2.0 ** -8 + 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (CPU or GPU)."""
    return t.detach().cpu().contiguous().view(torch.uint16).numpy().reshape(-1)


def oracle_quantized(w_t: torch.Tensor, codebook):
    """Oracle quantize + double-quant of a bf16 W^T: (codes_packed, absmax, e, sc, mu)."""
    codes, absmax = nf4.quantize_blockwise(bits(w_t), codebook)
    e, sc, mu = nf4.double_quant(absmax)
    return nf4.pack_codes(codes), absmax, e, sc, mu


# The other 4-bit data types the pages compare with NF4 (perplexity table of
# the QLoRA analysis: Int4, FP4 E2M1, FP4 E3M0), as 16-entry codebooks scaled
# to [-1, 1] with one exact zero: symmetric Int4 (-8 .. 7) / 8; the E2M1
# magnitudes {0.5, 1, 1.5, 2, 3, 4, 6} of both signs plus 8 as the 16th value,
# over 8; E3M0 (powers of two) 2^-6 .. 1 negative and 2^-7 .. 1 positive.
OTHER_CODEBOOKS = {
    "int4": (np.arange(16, dtype=np.float64) - 8) / 8.0,
    "fp4_e2m1": np.concatenate([-np.array([6, 4, 3, 2, 1.5, 1, 0.5]), [0.0],
                                np.array([0.5, 1, 1.5, 2, 3, 4, 6, 8])]) / 8.0,
    "fp4_e3m0": np.concatenate([-(2.0 ** np.arange(0, -7, -1)), [0.0], 2.0 ** np.arange(-7, 1)]),
}
OTHER_CODEBOOKS = {k: np.sort(v).astype(np.float32) for k, v in OTHER_CODEBOOKS.items()}


class Layer:
    """One seeded layer: W^T[o][h], X[M][h], dY[M][o], L1[h][r], L2[r][o]."""

    def __init__(self, M, h, o, r, s, seed=0, outlier_frac=0.0, codebook=None):
        self.M, self.h, self.o, self.r, self.s = M, h, o, r, s
        self.codebook = nf4.nf4_codebook() if codebook is None else np.asarray(codebook, np.float32)
        self.W_t = synth.weight_t(o, h, seed=seed, outlier_frac=outlier_frac)
        self.X = synth.activations(M, h, seed=seed, tag="X")
        self.dY = synth.activations(M, o, seed=seed, tag="dY")
        self.L1, self.L2 = synth.lora_factors(h, r, o, seed=seed)

    def oracle_weights(self):
        cp, absmax, e, sc, mu = oracle_quantized(self.W_t, self.codebook)
        wb = nf4.dequant(cp, e, sc, mu, self.codebook)
        wf = nf4.dequant(cp, e, sc, mu, self.codebook, out="f32")
        return (nf4.bf16_bits_to_f32(wb).reshape(self.o, self.h).astype(np.float64),
                wf.reshape(self.o, self.h).astype(np.float64))

    def f64(self, t):
        return t.float().numpy().astype(np.float64)
