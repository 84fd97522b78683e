"""CPU oracle: NF4 blockwise quantization, double quantization, dequantization
and the QLoRA frozen-base linear layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never imports, links or calls it, and this
module imports nothing from the product.

It is written to be checked by eye against the QLoRA pages, not to be fast:
plain numpy in the precision each step names, fp64 for the matmuls, one step
per function, in the order the pages give them.

Sources (QLoRA, Dettmers et al., NeurIPS 2023, as restated on the web pages):
  * diycv.top "QLoRA" walkthrough, "方法总览" (method overview):
      §1 blockwise quantization  - the Int8 absmax equation, block size 64;
      §2 NF4                     - the quantile-midpoint equation for q_i,
                                   normalisation to [-1, 1], separate halves
                                   with an exact zero;
      §3 double quantization     - the 0.5 and 0.127 bit/parameter equations,
                                   FP8 constants in blocks of 256, mean
                                   subtracted first;
    "关键公式" (key formulas) - the QLoRA linear-layer equation and the
      doubleDequant equation, plus the data-type table (NF4 storage, FP8
      first-level constants, FP32 second-level constants, BF16 compute);
    "训练" (training flow) - steps 1-2 (quantize, then double-quantize) and 5
      (backward passes through the frozen weight, gradients for LoRA only);
    "问题背景" (background) - the LoRA equation Y = XW + s X L1 L2 with
      L1 in R^{h x r}, L2 in R^{r x o}.
  * neura.market "QLoRA" analysis, "How It Works" - NF4 built from normal
    quantiles, asymmetric so that zero is exact; DQ with block 256 and mean
    subtraction.

Readings where the pages leave a step open:
  R2  packing: element 2k goes in the high nibble of byte k.
  R3  codebook truncation: the quantile-midpoint equation is infinite at the
      ends; the halves are built from normal quantiles at evenly spaced
      probabilities between 1/2 and DELTA = ((1 - 1/30) + (1 - 1/32)) / 2.
  R4  an all-zero block has absmax 0 and every code is the index of 0.0.
  R5  nearest code = number of fp32 midpoint thresholds strictly below
      x = fp32(w / absmax); a value exactly on a threshold takes the lower code.
  R6  one fp32 mean per tensor, computed from the exact fp64 sum.
  R7  FP8 E4M3 with round-to-nearest-even and saturation; each group of 256
      centred constants is scaled so that its absmax maps to 448.
  R8  a DQ group whose centred constants are all zero encodes as zeros.
  R9  output error metric: max|out - ref| / max|ref| per tensor.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtri  # standard normal quantile function Q(p)

__all__ = [
    "NF4_DELTA", "FP8_MAX", "nf4_codebook", "validate_codebook", "zero_index",
    "nearest_code_thresholds", "bf16_bits_to_f32", "f32_to_bf16_bits",
    "e4m3_values", "e4m3_decode", "e4m3_encode", "block_absmax",
    "quantize_blockwise", "pack_codes", "unpack_codes", "constant_mean",
    "double_quant", "dequant_constants", "dequant", "dequant_blocks", "lora_forward",
    "lora_backward", "rel_max_err", "constant_bits_per_param", "f64_to_bf16_bits", "merge_adapter",
    "philox4x32_10", "dropout_keep", "dropout_scale", "lora_forward_dropout", "lora_backward_dropout",
]

NF4_DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
FP8_MAX = 448.0          # largest finite E4M3 magnitude
_CHUNK = 1 << 20         # elements per chunk in the element-wise loops


# --------------------------------------------------------------------------
# Number formats (bf16 storage, FP8 E4M3 constants), from their definitions
# --------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 -> fp32 is exact: the 16 bf16 bits become the top half of the fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16, round to nearest, ties to even (the BF16 compute dtype).

    Drops the low 16 bits of the fp32 pattern; rounds up when they exceed half,
    and on an exact half when the kept part is odd.  NaN stays a quiet NaN.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep = u >> 16
    low = u & 0xFFFF
    up = (low > 0x8000) | ((low == 0x8000) & ((keep & 1) == 1))
    out = (keep + up.astype(np.uint64)).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if np.any(nan):
        out[nan] = (keep[nan] | 0x40).astype(np.uint16)
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 with ONE round-to-nearest (ties to even) of the exact value.

    Going through fp32 first could round twice (a value just above a bf16
    midpoint can land on the midpoint in fp32, whose tie then goes to even), so
    the fp32 route only supplies a candidate: the result is whichever of it and
    its two bf16 neighbours is nearest in exact fp64 distance, an even pattern
    on a tie.  Finite inputs only.
    """
    x = np.asarray(x, dtype=np.float64)
    assert np.all(np.isfinite(x)), "finite input expected"
    mag = np.abs(x)
    c = f32_to_bf16_bits(mag.astype(np.float32)).astype(np.int64)
    cands = np.stack([np.maximum(c - 1, 0), c, c + 1])               # positive patterns, increasing
    vals = bf16_bits_to_f32(cands.astype(np.uint16)).astype(np.float64)
    dist = np.abs(vals - mag[None])
    best = np.argmin(dist, axis=0)
    d_best = np.take_along_axis(dist, best[None], 0)[0]
    pick = np.take_along_axis(cands, best[None], 0)[0]
    # a tie between two neighbours goes to the even pattern
    for k in range(3):
        tie = (dist[k] == d_best) & (cands[k] != pick) & (cands[k] % 2 == 0)
        pick = np.where(tie, cands[k], pick)
    sign = (np.signbit(x)).astype(np.int64) << 15
    return (pick | sign).astype(np.uint16)


def e4m3_values() -> np.ndarray:
    """All 256 FP8 E4M3 codes decoded to fp64 (NaN at 0x7F and 0xFF).

    Format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent
    field 0 holds subnormals m * 2^-9; there is no infinity; the all-ones
    exponent with all-ones mantissa is NaN, so the largest finite value is
    1.75 * 2^8 = 448.
    """
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * m * 2.0 ** -9
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_values()
_E4M3_MAG = _E4M3[:0x7F]          # codes 0x00..0x7E: 0 .. 448, increasing


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 code -> fp32 (every finite E4M3 value is exact in fp32)."""
    return _E4M3[np.asarray(codes, dtype=np.uint8)].astype(np.float32)


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """fp32 -> FP8 E4M3: nearest finite value, ties to the even code,
    magnitudes beyond 448 saturate to 448; the sign bit is kept (so -0 -> 0x80).
    """
    y = np.asarray(y, dtype=np.float32)
    assert np.all(np.isfinite(y)), "E4M3 encode expects finite input"
    a = np.abs(y).astype(np.float64)
    hi = np.searchsorted(_E4M3_MAG, a, side="left")      # first magnitude >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    # a lies in [mag[lo], mag[hi]] unless it is above 448 (then it saturates).
    twice = 2.0 * a                                        # exact in fp64
    mid2 = _E4M3_MAG[lo] + _E4M3_MAG[hi]                   # exact in fp64
    pick_hi = (twice > mid2) | ((twice == mid2) & (hi % 2 == 0))
    mag_code = np.where(a >= _E4M3_MAG[hi], hi, np.where(pick_hi, hi, lo))
    mag_code = np.where(a <= 0.0, 0, mag_code)
    sign = (y.view(np.uint32) >> 31).astype(np.uint8)
    return (mag_code.astype(np.uint8) | (sign << 7)).astype(np.uint8)


# --------------------------------------------------------------------------
# NF4 data type (diycv.top §2 NF4; neura.market "How It Works")
# --------------------------------------------------------------------------

def nf4_codebook() -> np.ndarray:
    """The 16 NF4 code values, fp32, strictly increasing, in [-1, 1].

    Each half is built separately from standard-normal quantiles Q(p) at evenly
    spaced probabilities from DELTA down to 1/2 (reading R3): 9 points for the
    positive half and 8 for the negative half; the point p = 1/2 (Q = 0) is
    dropped from both and a single exact zero is added, which gives 7 negative
    values, 0 and 8 positive values.  The set is then divided by its largest
    value, so that it spans exactly [-1, 1].
    """
    pos = ndtri(np.linspace(NF4_DELTA, 0.5, 9))[:-1]      # 8 values > 0
    neg = -ndtri(np.linspace(NF4_DELTA, 0.5, 8))[:-1]     # 7 values < 0
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    v = v / v.max()
    return v.astype(np.float32)


def validate_codebook(q: np.ndarray) -> None:
    """A codebook is 16 finite, strictly increasing fp32 values with exactly one 0.0."""
    q = np.asarray(q, dtype=np.float32)
    assert q.shape == (16,), "codebook must have 16 entries (k = 4 bits)"
    assert np.all(np.isfinite(q)), "codebook must be finite"
    assert np.all(np.diff(q.astype(np.float64)) > 0), "codebook must be strictly increasing"
    assert int(np.sum(q == 0.0)) == 1, "codebook must hold exactly one zero"


def zero_index(q: np.ndarray) -> int:
    """Index of the exact zero, the code of an all-zero block (reading R4)."""
    return int(np.flatnonzero(np.asarray(q, dtype=np.float32) == 0.0)[0])


def nearest_code_thresholds(q: np.ndarray) -> np.ndarray:
    """t_j = fp32((q_j + q_{j+1}) / 2), j = 0..14: the midpoints between
    neighbouring codes (sum and halving are exact in fp64, one fp32 rounding)."""
    q64 = np.asarray(q, dtype=np.float32).astype(np.float64)
    return ((q64[:-1] + q64[1:]) / 2.0).astype(np.float32)


# --------------------------------------------------------------------------
# Blockwise absmax quantization (diycv.top §1, Int8 absmax equation; §2 NF4)
# --------------------------------------------------------------------------

def block_absmax(w_bits: np.ndarray, block: int = 64) -> np.ndarray:
    """c[b] = max over the b-th block of |w| (contiguous blocks of the flat
    tensor), fp32; exact because every bf16 magnitude is an fp32 value."""
    w = bf16_bits_to_f32(w_bits).reshape(-1, block)
    assert np.all(np.isfinite(w)), "weights must be finite"
    return np.max(np.abs(w), axis=1).astype(np.float32)


def quantize_blockwise(w_bits: np.ndarray, codebook: np.ndarray, block: int = 64):
    """Quantize a flat bf16 tensor to 4-bit codes with one absmax per block.

    Per block b: c = absmax (fp32); each element becomes x = fp32(w / c)
    (one IEEE round-to-nearest division), and its code is the number of
    midpoint thresholds t_j with x > t_j (reading R5), i.e. the nearest
    codebook value.  An all-zero block takes the index of 0.0 (R4).

    Returns (codes uint8 [n] one code per element, absmax fp32 [n / block]).
    """
    validate_codebook(codebook)
    w_bits = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    n = w_bits.size
    assert n % block == 0, "n must be a multiple of the block size"
    absmax = block_absmax(w_bits, block)
    t = nearest_code_thresholds(codebook)
    zi = zero_index(codebook)
    codes = np.empty(n, dtype=np.uint8)
    step = (_CHUNK // block) * block
    for s in range(0, n, step):
        e = min(n, s + step)
        w = bf16_bits_to_f32(w_bits[s:e]).reshape(-1, block)
        c = absmax[s // block:e // block]
        nz = c > 0
        out = np.full(w.shape, zi, dtype=np.uint8)
        x = w[nz] / c[nz, None]                         # fp32 / fp32 -> fp32, RN
        out[nz] = np.sum(x[:, :, None] > t[None, None, :], axis=2).astype(np.uint8)
        codes[s:e] = out.reshape(-1)
    return codes, absmax


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte; element 2k in the high nibble (R2)."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    assert codes.size % 2 == 0
    return ((codes[0::2] << 4) | (codes[1::2] & 0xF)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed >> 4
    out[1::2] = packed & 0xF
    return out


# --------------------------------------------------------------------------
# Double quantization (diycv.top §3; neura.market "How It Works")
# --------------------------------------------------------------------------

def _assert_exact_fp64_sum(c: np.ndarray) -> None:
    """Every absmax is a bf16 value (8 significant bits).  Their fp64 sum is
    exact, whatever the order, when the span from the largest to the smallest
    nonzero value's last significant bit, plus the carry bits of nb terms,
    fits in 53 bits."""
    nz = c[c > 0].astype(np.float64)
    if nz.size == 0:
        return
    e_hi = math.frexp(float(nz.max()))[1]
    e_lo = math.frexp(float(nz.min()))[1] - 8
    carry = math.ceil(math.log2(c.size)) + 1
    assert (e_hi - e_lo) + carry <= 53, "absmax spread too wide for an exact fp64 sum"


def constant_mean(absmax: np.ndarray) -> np.float32:
    """mu = fp32(fp64(sum of all first-level constants) / nb)  (R6)."""
    c = np.asarray(absmax, dtype=np.float32)
    _assert_exact_fp64_sum(c)
    total = float(np.sum(c.astype(np.float64)))
    return np.float32(total / float(c.size))


def double_quant(absmax: np.ndarray, dq_block: int = 256):
    """Quantize the fp32 first-level constants to FP8 E4M3 in groups of 256.

    mu = constant_mean(absmax); d = fp32(c - mu);
    dq_scale[g] = max over group g of |d|;
    y = fp32(d * fp32(448 / dq_scale[g]));  e = E4M3(y) (RN-even, saturating).
    A group with dq_scale = 0 encodes as zeros (R8).

    Returns (absmax_fp8 uint8 [nb], dq_scale fp32 [nb / 256], dq_mean fp32).
    """
    c = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nb = c.size
    assert nb % dq_block == 0, "number of blocks must be a multiple of the DQ block"
    mu = constant_mean(c)
    d = (c - mu).astype(np.float32)                       # fp32 subtraction, RN
    g = d.reshape(-1, dq_block)
    dq_scale = np.max(np.abs(g), axis=1).astype(np.float32)
    e = np.zeros(g.shape, dtype=np.uint8)
    ok = dq_scale > 0
    inv = (np.float32(FP8_MAX) / dq_scale[ok]).astype(np.float32)   # fp32 RN
    y = (g[ok] * inv[:, None]).astype(np.float32)                    # fp32 RN
    e[ok] = e4m3_encode(y)
    return e.reshape(-1), dq_scale, np.float32(mu)


def dequant_constants(absmax_fp8: np.ndarray, dq_scale: np.ndarray, dq_mean,
                      dq_block: int = 256) -> np.ndarray:
    """c' = fp32(fp32(E4M3(e) * fp32(dq_scale / 448)) + mu): the inner dequant
    of doubleDequant, three separately rounded fp32 operations (no FMA)."""
    step = (np.asarray(dq_scale, dtype=np.float32) / np.float32(FP8_MAX)).astype(np.float32)
    v = e4m3_decode(absmax_fp8).reshape(-1, dq_block)
    c = (v * step[:, None]).astype(np.float32)
    c = (c + np.float32(dq_mean)).astype(np.float32)
    return c.reshape(-1)


def dequant(codes_packed: np.ndarray, absmax_fp8: np.ndarray, dq_scale: np.ndarray,
            dq_mean, codebook: np.ndarray, block: int = 64, dq_block: int = 256,
            out: str = "bf16") -> np.ndarray:
    """doubleDequant: W'_i = bf16(fp32(q[code_i] * c'[b])) with c' from
    dequant_constants; ``out="f32"`` keeps the fp32 product (no bf16 rounding).

    Returns the flat tensor: uint16 bf16 bit patterns, or fp32.
    """
    cp = dequant_constants(absmax_fp8, dq_scale, dq_mean, dq_block)
    return dequant_blocks(codes_packed, cp, codebook, block, out)


def dequant_blocks(codes_packed: np.ndarray, cprime: np.ndarray, codebook: np.ndarray,
                   block: int = 64, out: str = "bf16") -> np.ndarray:
    """Outer dequant of doubleDequant for blocks whose constants c' are known:
    W'_i = bf16(fp32(q[code_i] * c'[b]))  (``out="f32"`` keeps the product)."""
    q = np.asarray(codebook, dtype=np.float32)
    cp = np.asarray(cprime, dtype=np.float32).reshape(-1)
    codes = unpack_codes(codes_packed)
    assert codes.size == cp.size * block
    v = (q[codes].reshape(-1, block) * cp[:, None]).astype(np.float32).reshape(-1)
    if out == "f32":
        return v
    assert out == "bf16"
    return f32_to_bf16_bits(v)


# --------------------------------------------------------------------------
# QLoRA linear layer (diycv.top "关键公式"; "问题背景" LoRA equation;
# "训练" step 5).  W is h x o; storage is W^T [o][h].
# --------------------------------------------------------------------------

def lora_forward(X: np.ndarray, Wt: np.ndarray, L1: np.ndarray, L2: np.ndarray, s: float):
    """T = X L1;  Y = X W + s T L2, with W = Wt^T, all in fp64.  Returns (Y, T)."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(Wt, dtype=np.float64).T
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    T = X @ L1
    Y = X @ W + s * (T @ L2)
    return Y, T


def lora_backward(X: np.ndarray, dY: np.ndarray, Wt: np.ndarray, L1: np.ndarray,
                  L2: np.ndarray, s: float):
    """Gradients of <Y, dY> for Y = X W + s X L1 L2 with W frozen (no dW):
         U = dY L2^T;  dX = dY W^T + s U L1^T;  dL1 = s X^T U;  dL2 = s T^T dY.
    All fp64.  Returns (dX, dL1, dL2, U, T)."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    W = np.asarray(Wt, dtype=np.float64).T
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    T = X @ L1
    U = dY @ L2.T
    dX = dY @ W.T + s * (U @ L1.T)
    dL1 = s * (X.T @ U)
    dL2 = s * (T.T @ dY)
    return dX, dL1, dL2, U, T


def merge_adapter(Wp_bits: np.ndarray, L1: np.ndarray, L2: np.ndarray, s: float) -> np.ndarray:
    """Merge of the trained adapter into the 16-bit dequantized base (QLoRA
    glossary, pitfalls entry: into the bf16 dequantized weight, never into the
    4-bit codes): W_m = W' + s L1 L2, stored like the weight as W_m^T[o][h].
    W' (bf16 bits, [o][h]) is widened exactly, the sum is formed in fp64 and
    rounded once to bf16.  Returns uint16 bf16 bits [o][h]."""
    Wp = bf16_bits_to_f32(np.asarray(Wp_bits)).astype(np.float64)
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    o, h = L2.shape[1], L1.shape[0]
    v = Wp.reshape(o, h) + s * (L1 @ L2).T
    return f64_to_bf16_bits(v)


def rel_max_err(out: np.ndarray, ref: np.ndarray) -> float:
    """R9: max|out - ref| / max|ref| over one tensor."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(out - ref))) if ref.size else 0.0
    return num / den if den > 0 else num


# --------------------------------------------------------------------------
# LoRA dropout on the adapter input (diycv.top "训练与推理流程": LoRA dropout
# 0.1 for 7B/13B and 0.05 for 33B/65B, on all linear layers).  The pages give
# the rate only; the readings here: inverted dropout of the adapter's input X
# (the base path keeps X), a keep decision per element of X drawn from the
# counter-based generator Philox4x32-10, and the fp32 scale 1 / (1 - p).
# --------------------------------------------------------------------------

_PHILOX_M = (0xD2511F53, 0xCD9E8D57)       # round multipliers
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)       # key increments (Weyl sequence)
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counter, key):
    """Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
    numbers: as easy as 1, 2, 3", SC 2011).  counter: four uint32 arrays (one
    element per draw), key: two uint32 values.  Each round multiplies words 0
    and 2 by the two constants into 64-bit products, and the new words are
    (hi(w2*M1) ^ w1 ^ k0, lo(w2*M1), hi(w0*M0) ^ w3 ^ k1, lo(w0*M0)); the key
    advances by the Weyl constants between rounds.  Returns four uint32 arrays."""
    c = [np.asarray(v, dtype=np.uint64) & _U32 for v in counter]
    k0, k1 = np.uint64(key[0]) & _U32, np.uint64(key[1]) & _U32
    for rnd in range(10):
        if rnd:
            k0 = (k0 + np.uint64(_PHILOX_W[0])) & _U32
            k1 = (k1 + np.uint64(_PHILOX_W[1])) & _U32
        p0 = c[0] * np.uint64(_PHILOX_M[0])
        p1 = c[2] * np.uint64(_PHILOX_M[1])
        c = [((p1 >> np.uint64(32)) ^ c[1] ^ k0) & _U32, p1 & _U32,
             ((p0 >> np.uint64(32)) ^ c[3] ^ k1) & _U32, p0 & _U32]
    return [v.astype(np.uint32) for v in c]


def dropout_threshold(p: float) -> int:
    """An element is dropped when its 32-bit draw is below floor(p * 2^32),
    with p the fp32 value of the rate (as it is passed to the library)."""
    p32 = float(np.float32(p))
    assert 0.0 <= p32 < 1.0
    return min(int(math.floor(p32 * 4294967296.0)), 0xFFFFFFFF)


def dropout_keep(M: int, h: int, p: float, seed: int) -> np.ndarray:
    """Keep mask of the adapter input X [M][h]: element i = m h + k takes word
    i % 4 of Philox4x32-10 at counter (i // 4 low 32 bits, i // 4 high 32 bits,
    0, 0) under key (seed low 32 bits, seed high 32 bits), and is kept when
    that word is at least dropout_threshold(p)."""
    i = np.arange(M * h, dtype=np.uint64)
    blk = i >> np.uint64(2)
    zeros = np.zeros_like(blk)
    words = philox4x32_10([blk & _U32, blk >> np.uint64(32), zeros, zeros],
                          (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    w = np.choose((i & np.uint64(3)).astype(np.int64), words)
    return (w >= np.uint32(dropout_threshold(p))).reshape(M, h)


def dropout_scale(p: float) -> np.float32:
    """The inverted-dropout scale, fp32(1 / (1 - p)) with fp32 operations."""
    return np.float32(1.0) / (np.float32(1.0) - np.float32(p))


def lora_forward_dropout(X, Wt, L1, L2, s, keep, scale):
    """Y = X W + s T L2 with T = scale (X * keep) L1: dropout on the adapter
    input only; all fp64.  Returns (Y, T)."""
    X = np.asarray(X, dtype=np.float64)
    Xd = X * np.asarray(keep, dtype=np.float64)
    T = float(scale) * (Xd @ np.asarray(L1, dtype=np.float64))
    Y = X @ np.asarray(Wt, dtype=np.float64).T + s * (T @ np.asarray(L2, dtype=np.float64))
    return Y, T


def lora_backward_dropout(X, dY, Wt, L1, L2, s, keep, scale):
    """Gradients of <Y, dY> for lora_forward_dropout (W frozen):
         U = dY L2^T;  dX = dY W^T + s scale keep * (U L1^T);
         dL1 = s scale (X * keep)^T U;  dL2 = s T^T dY.
    All fp64.  Returns (dX, dL1, dL2, U, T)."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    W = np.asarray(Wt, dtype=np.float64).T
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    kp = np.asarray(keep, dtype=np.float64)
    sc = float(scale)
    Xd = X * kp
    T = sc * (Xd @ L1)
    U = dY @ L2.T
    dX = dY @ W.T + s * sc * kp * (U @ L1.T)
    dL1 = s * sc * (Xd.T @ U)
    dL2 = s * (T.T @ dY)
    return dX, dL1, dL2, U, T


# --------------------------------------------------------------------------
# Storage accounting (diycv.top §3, the 0.5 and 0.127 bit/parameter equations)
# --------------------------------------------------------------------------

def constant_bits_per_param(block: int = 64, dq_block: int = 256, const_bits: int = 32,
                            fp8_bits: int = 8, double_quantized: bool = True) -> float:
    """Bits of quantization constants per weight.

    Without DQ: one const_bits constant per block.  With DQ: one fp8_bits code
    per block, plus one const_bits second-level constant per dq_block blocks.
    """
    if not double_quantized:
        return const_bits / block
    return fp8_bits / block + const_bits / (block * dq_block)
