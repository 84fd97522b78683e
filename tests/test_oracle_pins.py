"""Pins of the CPU oracle against what the QLoRA pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers the
pages print, closed forms, format definitions, textbook values, library
routines, brute force on tiny inputs, or invariants.  A plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
tie rule) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nf4
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


# ---------------------------------------------------------------- quantiles

def test_normal_quantile_textbook_values():
    # Q(0.975) = 1.959963984540054 (two-sided 95% z value), Q(1/2) = 0,
    # Q(Phi(1)) = 1 with Phi from the error function.
    from scipy.special import ndtri
    assert abs(ndtri(0.975) - 1.959963984540054) < 1e-14
    assert ndtri(0.5) == 0.0
    phi1 = 0.5 * math.erfc(-1.0 / math.sqrt(2.0))
    assert abs(ndtri(phi1) - 1.0) < 1e-12
    for p in (0.51, 0.6, 0.75, 0.9, nf4.NF4_DELTA):
        z = ndtri(p)
        assert abs(0.5 * math.erfc(-z / math.sqrt(2.0)) - p) < 1e-15


# ---------------------------------------------------------------- codebook

def test_codebook_shape_and_range():
    # NF4 page facts: 2^k = 16 values, normalised to [-1, 1], halves built
    # separately with one exact zero ("asymmetric to include zero exactly").
    q = nf4.nf4_codebook()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q.astype(np.float64)) > 0)
    assert q[0] == -1.0 and q[-1] == 1.0
    assert np.sum(q == 0.0) == 1 and nf4.zero_index(q) == 7
    assert np.sum(q < 0) == 7 and np.sum(q > 0) == 8
    nf4.validate_codebook(q)


def test_codebook_is_equal_probability_quantiles():
    # Undo the normalisation and map each code back through the normal CDF:
    # the positive codes must sit at evenly spaced probabilities (step
    # (DELTA - 1/2) / 8) and the negative ones at step (DELTA - 1/2) / 7,
    # the quantile construction's defining property.
    from scipy.special import ndtri
    q = nf4.nf4_codebook().astype(np.float64)
    zmax = ndtri(nf4.NF4_DELTA)
    cdf = lambda z: 0.5 * math.erfc(-z / math.sqrt(2.0))  # noqa: E731
    pos = [cdf(v * zmax) for v in q[8:]]
    neg = [cdf(-v * zmax) for v in q[:7]]
    dp = (nf4.NF4_DELTA - 0.5) / 8
    dn = (nf4.NF4_DELTA - 0.5) / 7
    assert np.allclose(np.diff(pos), dp, atol=2e-7)
    assert abs(pos[0] - 0.5 - dp) < 2e-7 and abs(pos[-1] - nf4.NF4_DELTA) < 2e-7
    assert np.allclose(np.diff(neg[::-1]), dn, atol=2e-7)
    assert abs(neg[-1] - 0.5 - dn) < 2e-7 and abs(neg[0] - nf4.NF4_DELTA) < 2e-7


def test_codebook_frozen_copy():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "nf4_codebook.txt")) if not l.startswith("#")]
    frozen = np.array([int(r[0], 16) for r in rows], dtype=np.uint32).view(np.float32)
    assert np.array_equal(frozen.view(np.uint32), nf4.nf4_codebook().view(np.uint32))


def test_codebook_validation_rejects_bad_tables():
    q = nf4.nf4_codebook()
    with pytest.raises(AssertionError):
        nf4.validate_codebook(q[::-1])
    bad = q.copy(); bad[7] = 1e-3
    with pytest.raises(AssertionError):
        nf4.validate_codebook(bad)
    with pytest.raises(AssertionError):
        nf4.validate_codebook(q[:15])


# ---------------------------------------------------------------- storage accounting

def test_constant_overhead_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "overhead.json")))
    without = nf4.constant_bits_per_param(g["block"], g["dq_block"], double_quantized=False)
    with_dq = nf4.constant_bits_per_param(g["block"], g["dq_block"], double_quantized=True)
    assert without == g["bits_without_dq"]
    assert round(with_dq, g["printed_decimals"]) == g["bits_with_dq_printed"]
    assert with_dq == 0.126953125                  # 8/64 + 32/16384 exactly
    saving = without - with_dq
    assert round(saving, g["printed_decimals"]) == g["saving_printed"]
    gb = g["params_65b"] * saving / 8 / 1e9
    assert abs(gb - g["saving_gb_65b_printed"]) / g["saving_gb_65b_printed"] < g["saving_gb_tolerance"]


# ---------------------------------------------------------------- number formats

def test_bf16_rounding_matches_library():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    # exact ties and near-ties around them
    base = rng.integers(0, 2**31, 5000, dtype=np.uint64).astype(np.uint32) & 0x7F7F0000
    ties = np.concatenate([base | 0x8000, base | 0x18000, base | 0x7FFF, base | 0x8001]).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, 3.3895314e38])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(nf4.f32_to_bf16_bits(x), ref)
    back = nf4.bf16_bits_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_e4m3_format_closed_forms():
    v = nf4.e4m3_values()
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.sum(np.isfinite(v)) == 254
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9 and v[0x08] == 2.0 ** -6
    assert v[0x38] == 1.0 and v[0x00] == 0.0 and v[0x80] == 0.0 and math.copysign(1, v[0x80]) < 0
    mags = v[:0x7F]
    assert np.all(np.diff(mags) > 0)
    assert np.array_equal(v[0x80:0xFF], -mags)


def test_e4m3_encode_matches_library_and_ties_to_even():
    v = nf4.e4m3_values()
    finite = [c for c in range(256) if np.isfinite(v[c])]
    codes = np.array(finite, dtype=np.uint8)
    assert np.array_equal(nf4.e4m3_encode(nf4.e4m3_decode(codes)), codes)
    mags = v[:0x7F]
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)     # exact in fp32
    enc = nf4.e4m3_encode(mids)
    lo = np.arange(0x7E)
    assert np.array_equal(enc, np.where(lo % 2 == 0, lo, lo + 1))
    nudge_up = np.nextafter(mids, np.float32(np.inf))
    nudge_dn = np.nextafter(mids, np.float32(0))
    assert np.array_equal(nf4.e4m3_encode(nudge_up), lo + 1)
    assert np.array_equal(nf4.e4m3_encode(nudge_dn), lo)
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.uniform(-448, 448, 300000),
                        rng.standard_normal(100000) * 2.0 ** rng.uniform(-12, 8, 100000),
                        mids, -mids, nudge_up, nudge_dn]).astype(np.float32)
    y = np.clip(y, -448, 448)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_encode(y), ref)
    # saturation (the finite-only variant of the format)
    assert np.all(nf4.e4m3_encode(np.float32([449.0, 1e30, 464.0])) == 0x7E)
    assert np.all(nf4.e4m3_encode(np.float32([-449.0, -1e30])) == 0xFE)


# ---------------------------------------------------------------- blockwise NF4 quantization

def _exact_nearest(w, c, q):
    """Brute force in exact rationals: all codes j minimising |w/c - q_j|."""
    x = Fraction(float(w)) / Fraction(float(c))
    d = [abs(x - Fraction(float(v))) for v in q]
    m = min(d)
    return {j for j, dj in enumerate(d) if dj == m}, x


def test_quantize_agrees_with_exact_nearest_code():
    q = nf4.nf4_codebook()
    mids = [(Fraction(float(q[j])) + Fraction(float(q[j + 1]))) / 2 for j in range(15)]
    rng = np.random.default_rng(3)
    w = _bf16(rng.standard_normal(64 * 40) * 0.02)
    codes, absmax = nf4.quantize_blockwise(w, q)
    wf = nf4.bf16_bits_to_f32(w)
    near_mid = 0
    for i in range(w.size):
        c = absmax[i // 64]
        best, x = _exact_nearest(wf[i], c, q)
        if codes[i] in best:
            continue
        # Only allowed where fp32 rounding of x or of the threshold decides:
        # x within 2^-23 |x| + 2^-24 of a true midpoint, and the code adjacent.
        gap = min(abs(x - m) for m in mids)
        assert gap <= Fraction(abs(float(x))) * Fraction(1, 2**23) + Fraction(1, 2**24), (i, float(x))
        assert min(abs(int(codes[i]) - b) for b in best) == 1
        near_mid += 1
    assert near_mid <= 2


def test_quantize_midpoint_ties_take_lower_code():
    # R5: an element whose fp32 ratio lands exactly on a threshold takes the
    # lower code; the next bf16 value above takes the upper one.  The uniform
    # codebook (j - 7) / 8 has thresholds (2i + 1) / 16 that are bf16 values,
    # and absmax 1.0 makes x = w exactly.
    qu = ((np.arange(16) - 7) / 8.0).astype(np.float32)
    t = nf4.nearest_code_thresholds(qu)
    assert np.array_equal(t, ((np.arange(15) * 2 - 13) / 16.0).astype(np.float32))
    for j in range(15):
        on = _bf16([t[j]])
        above = (on.astype(np.int32) + (1 if t[j] > 0 else -1)).astype(np.uint16)
        blk = np.concatenate([on, above, _bf16([1.0]), _bf16(np.zeros(61))])
        codes, _ = nf4.quantize_blockwise(blk, qu)
        assert codes[0] == j and codes[1] == j + 1, j


def test_quantize_absmax_element_and_codebook_values():
    q = nf4.nf4_codebook()
    rng = np.random.default_rng(4)
    for c in (0.0371, 1.0, 3.5e-5, 0.16, 2.0 ** -20):
        vals = [float(v) * c for v in q] + list(rng.uniform(-c, c, 48))
        blk = _bf16(vals)
        cb = nf4.bf16_bits_to_f32(_bf16([c]))[0]
        codes, absmax = nf4.quantize_blockwise(blk, q)
        assert absmax[0] == cb
        assert np.array_equal(codes[:16], np.arange(16))     # bf16(q_j c) -> code j
    neg = _bf16([-0.5] + [0.25] * 63)
    codes, absmax = nf4.quantize_blockwise(neg, q)
    assert absmax[0] == 0.5 and codes[0] == 0


def test_quantize_all_zero_block_and_signed_zero():
    # R4: an all-zero block (either sign of zero) has absmax 0 and every code
    # is the index of 0.0; after double quantization it dequantizes to zeros
    # only if its reconstructed constant times 0.0 is zero, which holds for
    # any finite constant.
    q = nf4.nf4_codebook()
    rest = synth.weight_t(1, 64 * 254, seed=5).view(torch.uint16).numpy().reshape(-1)
    blk = np.concatenate([np.zeros(64, np.uint16), np.full(64, 0x8000, np.uint16), rest])
    codes, absmax = nf4.quantize_blockwise(blk, q)
    assert np.all(absmax[:2] == 0) and np.all(codes[:128] == 7)
    e, sc, mu = nf4.double_quant(absmax)
    w = nf4.bf16_bits_to_f32(nf4.dequant(nf4.pack_codes(codes), e, sc, mu, q))
    assert np.all(w[:128] == 0)


def test_uniform_codebook_reduces_to_absmax_rounding():
    # With the uniform codebook (j - 7) / 8 the nearest code is the absmax
    # rounding of the Int8 example with 127 replaced by 8: code = rint(8 x) + 7,
    # clamped at the bottom code.
    qu = ((np.arange(16) - 7) / 8.0).astype(np.float32)
    rng = np.random.default_rng(5)
    w = _bf16(rng.standard_normal(64 * 200))
    codes, absmax = nf4.quantize_blockwise(w, qu)
    x = (nf4.bf16_bits_to_f32(w).reshape(-1, 64) / absmax[:, None]).astype(np.float32).reshape(-1)
    k = 8.0 * x.astype(np.float64)
    frac = np.abs(k - np.floor(k) - 0.5)
    ok = frac > 1e-6                                     # skip exact ties
    ref = np.clip(np.rint(k) + 7, 0, 15)
    assert np.array_equal(codes[ok], ref[ok].astype(np.uint8))
    assert ok.mean() > 0.99


def test_pack_nibble_order():
    assert nf4.pack_codes(np.array([1, 2, 15, 0], np.uint8)).tolist() == [0x12, 0xF0]
    c = np.random.default_rng(6).integers(0, 16, 1000).astype(np.uint8)
    assert np.array_equal(nf4.unpack_codes(nf4.pack_codes(c)), c)


# ---------------------------------------------------------------- double quantization

def test_dq_constant_constants_are_exact():
    c = np.full(512, 0.0625, np.float32)
    e, sc, mu = nf4.double_quant(c)
    assert mu == np.float32(0.0625) and np.all(sc == 0) and np.all(e == 0)
    assert np.all(nf4.dequant_constants(e, sc, mu) == np.float32(0.0625))


def test_dq_mean_is_centre_of_symmetric_constants():
    a, d = 0.03125, 0.0078125
    c = np.array([a - d, a + d] * 256, np.float32)
    e, sc, mu = nf4.double_quant(c)
    assert mu == np.float32(a)
    assert np.all(sc == np.float32(d))
    assert np.all(e[0::2] == 0xFE) and np.all(e[1::2] == 0x7E)   # -448, +448
    assert np.array_equal(nf4.dequant_constants(e, sc, mu), c)


def test_dq_extreme_maps_to_448_and_error_bound():
    rng = np.random.default_rng(7)
    w = synth.weight_t(64, 1024, seed=3, outlier_frac=0.001)
    bits = w.view(torch.uint16).numpy().reshape(-1)
    _, c = nf4.quantize_blockwise(bits, nf4.nf4_codebook())
    e, sc, mu = nf4.double_quant(c)
    dec = nf4.e4m3_decode(e).reshape(-1, 256)
    assert np.all(np.max(np.abs(dec), axis=1) == 448.0)
    cp = nf4.dequant_constants(e, sc, mu).astype(np.float64)
    step = (sc.astype(np.float64) / 448.0)[:, None]
    y = ((c.astype(np.float64) - float(mu)).reshape(-1, 256)) / step
    half = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10)           # E4M3 half-step
    slop = 8 * 2.0 ** -24 * (np.abs(c.reshape(-1, 256)) + abs(float(mu)) + 448 * step)
    err = np.abs(cp.reshape(-1, 256) - c.reshape(-1, 256))
    assert np.all(err <= half * step + slop)
    assert rng is not None


def test_dq_exact_sum_guard():
    c = np.full(256, 1.0, np.float32)
    c[0] = 2.0 ** -60
    with pytest.raises(AssertionError):
        nf4.double_quant(c)


# ---------------------------------------------------------------- dequant

def _quantize_all(w_t):
    q = nf4.nf4_codebook()
    bits = w_t.view(torch.uint16).numpy().reshape(-1)
    codes, c = nf4.quantize_blockwise(bits, q)
    e, sc, mu = nf4.double_quant(c)
    return q, bits, codes, c, e, sc, mu


def test_dequant_round_trip_error_and_layout():
    o, h = 64, 512
    w_t = synth.weight_t(o, h, seed=11)
    q, bits, codes, c, e, sc, mu = _quantize_all(w_t)
    wp = nf4.bf16_bits_to_f32(nf4.dequant(nf4.pack_codes(codes), e, sc, mu, q)).reshape(o, h)
    w = w_t.float().numpy()
    cp = nf4.dequant_constants(e, sc, mu)
    # per element: |W' - W| <= c * (largest half gap of the codebook) + |c' - c| + bf16 rounding
    half_gap = float(np.max(np.diff(q.astype(np.float64)))) / 2
    bound = (c * half_gap + np.abs(cp - c) + 2.0 ** -8 * np.abs(cp)).repeat(64).reshape(o, h)
    assert np.all(np.abs(wp - w) <= bound * (1 + 1e-6))
    rel = np.sqrt(np.mean((wp - w) ** 2) / np.mean(w ** 2))
    assert 0.03 < rel < 0.15


def test_dequant_zero_code_is_zero_and_requantize_is_idempotent():
    o, h = 32, 512
    w_t = synth.weight_t(o, h, seed=12)
    q, bits, codes, c, e, sc, mu = _quantize_all(w_t)
    wp_bits = nf4.dequant(nf4.pack_codes(codes), e, sc, mu, q)
    wp = nf4.bf16_bits_to_f32(wp_bits)
    assert np.all(wp[codes == 7] == 0)
    codes2, _ = nf4.quantize_blockwise(wp_bits, q)
    cb = codes.reshape(-1, 64)
    has_extreme = np.any((cb == 0) | (cb == 15), axis=1)
    cp = nf4.dequant_constants(e, sc, mu)
    sel = has_extreme & (cp > 0)
    assert sel.mean() > 0.9
    assert np.array_equal(codes2.reshape(-1, 64)[sel], cb[sel])


def test_dequant_f32_mode_is_unrounded_product():
    o, h = 64, 256
    w_t = synth.weight_t(o, h, seed=13)
    q, bits, codes, c, e, sc, mu = _quantize_all(w_t)
    f = nf4.dequant(nf4.pack_codes(codes), e, sc, mu, q, out="f32")
    b = nf4.bf16_bits_to_f32(nf4.dequant(nf4.pack_codes(codes), e, sc, mu, q))
    assert np.array_equal(b, torch.from_numpy(f).to(torch.bfloat16).float().numpy())


def test_single_level_constants_return_each_block_absmax_exactly():
    # Without double quantization the block constant is the block absmax
    # itself (a bf16 value), so the element that sets it (q = +1 or -1)
    # dequantizes to exactly its own value; every other element stays within
    # half the widest codebook gap of it, plus one bf16 rounding.
    o, h = 64, 512
    w_t = synth.weight_t(o, h, seed=21, outlier_frac=0.002)
    q = nf4.nf4_codebook()
    bits = w_t.view(torch.uint16).numpy().reshape(-1)
    codes, c = nf4.quantize_blockwise(bits, q)
    wp = nf4.bf16_bits_to_f32(nf4.dequant_blocks(nf4.pack_codes(codes), c, q)).reshape(-1, 64)
    w = nf4.bf16_bits_to_f32(bits).reshape(-1, 64)
    rows = np.arange(w.shape[0])
    at = np.argmax(np.abs(w), axis=1)
    assert np.array_equal(wp[rows, at], w[rows, at])
    half_gap = float(np.max(np.diff(q.astype(np.float64)))) / 2
    bound = (c * (half_gap + 2.0 ** -8))[:, None]
    assert np.all(np.abs(wp - w) <= bound * (1 + 1e-6))
    # the double-quantized constants are not the absmax, so there it is not exact
    e, sc, mu = nf4.double_quant(c)
    assert np.mean(nf4.dequant_constants(e, sc, mu) != c) > 0.5


def test_f64_to_bf16_rounds_once():
    # fp32-representable inputs: the library's fp32 -> bf16 conversion
    x = np.random.default_rng(3).standard_normal(20000).astype(np.float32) * 3.0
    assert np.array_equal(nf4.f64_to_bf16_bits(x.astype(np.float64)), _bf16(x))
    # 1 (0x3F80) and 1 + 2^-7 (0x3F81) have the midpoint 1 + 2^-8; just above it
    # the exact value must go up although its fp32 rounding is the midpoint
    # itself, whose tie would go to the even 0x3F80
    mid = 1.0 + 2.0 ** -8
    got = nf4.f64_to_bf16_bits(np.array([mid + 2.0 ** -40, mid - 2.0 ** -40, mid, -(mid + 2.0 ** -40)]))
    assert list(got) == [0x3F81, 0x3F80, 0x3F80, 0xBF81]
    # odd lower neighbour: the tie goes up to the even pattern
    mid2 = 1.0 + 3 * 2.0 ** -8
    assert nf4.f64_to_bf16_bits(np.array([mid2]))[0] == 0x3F82


def test_merge_adapter_brute_force_and_special_cases():
    # tiny case by explicit loops: W_m^T[n][k] = W'^T[n][k] + s sum_j L1[k][j] L2[j][n]
    rng = np.random.default_rng(8)
    o, h, r, s = 3, 4, 2, 0.75
    Wp = _bf16(rng.standard_normal((o, h)) * 0.02)
    L1 = rng.standard_normal((h, r)) * 0.1
    L2 = rng.standard_normal((r, o)) * 0.1
    got = nf4.merge_adapter(Wp, L1, L2, s)
    wp = nf4.bf16_bits_to_f32(Wp).astype(np.float64)
    for n in range(o):
        for k in range(h):
            v = wp[n, k] + s * sum(L1[k, j] * L2[j, n] for j in range(r))
            assert got[n, k] == nf4.f64_to_bf16_bits(np.array([v]))[0]
    # no adapter: the merged weight is the base itself, bit for bit
    assert np.array_equal(nf4.merge_adapter(Wp, L1, np.zeros((r, o)), s), Wp)
    # the merged layer reproduces the adapter forward up to the bf16 rounding of W_m
    X, dY, Wt, L1b, L2b = _layer(seed=4, M=32, h=256, o=128, r=8)
    Wb = _bf16(Wt)
    Y, _ = nf4.lora_forward(X, nf4.bf16_bits_to_f32(Wb).astype(np.float64), L1b, L2b, 2.0)
    Wm = nf4.bf16_bits_to_f32(nf4.merge_adapter(Wb, L1b, L2b, 2.0)).astype(np.float64)
    assert nf4.rel_max_err(X @ Wm.T, Y) <= 2.0 ** -8


# ---------------------------------------------------------------- LoRA dropout

def test_philox_known_answer_vectors():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    assert len(rows) == 3
    for row in rows:
        v = [int(x, 16) for x in row]
        out = nf4.philox4x32_10([np.array([c], dtype=np.uint32) for c in v[:4]], (v[4], v[5]))
        assert [int(w[0]) for w in out] == v[6:], row


def test_dropout_mask_rate_and_threshold():
    M, h = 256, 1024
    for p in (0.05, 0.1, 0.5):
        keep = nf4.dropout_keep(M, h, p, seed=1234)
        n = keep.size
        # binomial: the kept fraction is within 6 standard deviations of 1 - p
        assert abs(keep.mean() - (1 - p)) <= 6 * math.sqrt(p * (1 - p) / n)
        # neighbouring elements (same Philox call, or consecutive calls) are independent
        a, b = keep.reshape(-1)[:-1].astype(float), keep.reshape(-1)[1:].astype(float)
        assert abs(np.corrcoef(a, b)[0, 1]) < 6 / math.sqrt(n)
    assert nf4.dropout_keep(4, 64, 0.0, seed=7).all()
    # floor(p 2^32) of the fp32 rate: fp32(0.1) = 13421773 / 2^27
    assert nf4.dropout_threshold(0.1) == (13421773 * 2 ** 5) and nf4.dropout_threshold(0.0) == 0
    # the seed changes the mask; the same seed gives the same mask
    assert not np.array_equal(nf4.dropout_keep(8, 256, 0.1, 1), nf4.dropout_keep(8, 256, 0.1, 2))
    assert np.array_equal(nf4.dropout_keep(8, 256, 0.1, 3), nf4.dropout_keep(8, 256, 0.1, 3))
    # element i draws word i % 4 of the Philox call at counter i // 4
    w = nf4.philox4x32_10([np.array([1], np.uint32), np.array([0], np.uint32), np.array([0], np.uint32),
                           np.array([0], np.uint32)], (99, 0))
    keep = nf4.dropout_keep(1, 8, 0.5, seed=99).reshape(-1)
    assert [bool(keep[4 + j]) for j in range(4)] == [int(w[j][0]) >= 2 ** 31 for j in range(4)]
    assert nf4.dropout_scale(0.1) == np.float32(1) / np.float32(0.9)


def test_dropout_zero_rate_is_plain_lora_and_backward_matches_finite_differences():
    X, dY, Wt, L1, L2 = _layer(seed=6, M=8, h=64, o=64, r=4)
    ones = np.ones_like(X, dtype=bool)
    Y0, T0 = nf4.lora_forward(X, Wt, L1, L2, 0.5)
    Y1, T1 = nf4.lora_forward_dropout(X, Wt, L1, L2, 0.5, ones, np.float32(1.0))
    assert np.allclose(Y0, Y1, rtol=0, atol=1e-12) and np.allclose(T0, T1, rtol=0, atol=1e-12)
    keep = nf4.dropout_keep(8, 64, 0.25, seed=5)
    sc = nf4.dropout_scale(0.25)
    dX, dL1, dL2, _, _ = nf4.lora_backward_dropout(X, dY, Wt, L1, L2, 0.5, keep, sc)
    f = lambda X_, L1_, L2_: float(np.sum(nf4.lora_forward_dropout(X_, Wt, L1_, L2_, 0.5, keep, sc)[0] * dY))
    eps = 1e-6
    for (arr, grad, which) in ((X, dX, 0), (L1, dL1, 1), (L2, dL2, 2)):
        rng = np.random.default_rng(which)
        for _ in range(6):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            a, b = arr.copy(), arr.copy()
            a[idx] += eps
            b[idx] -= eps
            args_a = [X, L1, L2]
            args_b = [X, L1, L2]
            args_a[which], args_b[which] = a, b
            fd = (f(*args_a) - f(*args_b)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx)
    # dropped inputs receive only the base gradient
    dXb = dY @ Wt
    assert np.allclose(dX[~keep], dXb[~keep], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- linear layer

def _layer(seed=0, M=16, h=256, o=256, r=8):
    X = synth.activations(M, h, seed=seed).double().numpy()
    dY = synth.activations(M, o, seed=seed, tag="dY").double().numpy()
    L1, L2 = synth.lora_factors(h, r, o, seed=seed)
    Wt = synth.weight_t(o, h, seed=seed).double().numpy()
    return X, dY, Wt, L1.double().numpy(), L2.double().numpy()


def test_forward_brute_force_tiny():
    rng = np.random.default_rng(8)
    M, h, o, r, s = 3, 5, 4, 2, 0.75
    X, Wt, L1, L2 = (rng.standard_normal(sh) for sh in ((M, h), (o, h), (h, r), (r, o)))
    Y, T = nf4.lora_forward(X, Wt, L1, L2, s)
    for m in range(M):
        for j in range(o):
            base = sum(X[m][i] * Wt[j][i] for i in range(h))
            lora = sum(sum(X[m][i] * L1[i][k] for i in range(h)) * L2[k][j] for k in range(r))
            assert abs(Y[m][j] - (base + s * lora)) < 1e-12


def test_backward_matches_finite_differences():
    X, dY, Wt, L1, L2 = _layer()
    s = 2.0
    dX, dL1, dL2, U, T = nf4.lora_backward(X, dY, Wt, L1, L2, s)
    f = lambda X_, L1_, L2_: float(np.sum(nf4.lora_forward(X_, Wt, L1_, L2_, s)[0] * dY))  # noqa: E731
    rng = np.random.default_rng(9)
    eps = 1e-6
    for name, arr, grad in (("X", X, dX), ("L1", L1, dL1), ("L2", L2, dL2)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            args = {"X": X, "L1": L1, "L2": L2}
            p = arr.copy(); p[idx] += eps
            m = arr.copy(); m[idx] -= eps
            fp = f(*[p if k == name else args[k] for k in ("X", "L1", "L2")])
            fm = f(*[m if k == name else args[k] for k in ("X", "L1", "L2")])
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx)


def test_zero_adapter_reduces_to_plain_matmul():
    X, dY, Wt, L1, L2 = _layer(seed=1)
    Y, _ = nf4.lora_forward(X, Wt, np.zeros_like(L1), L2, 2.0)
    assert np.array_equal(Y, X @ Wt.T)
    dX, dL1, dL2, _, _ = nf4.lora_backward(X, dY, Wt, L1, np.zeros_like(L2), 2.0)
    assert np.array_equal(dX, dY @ Wt) and not np.any(dL1)
    Y0, _ = nf4.lora_forward(X, Wt, L1, L2, 0.0)
    Y1, _ = nf4.lora_forward(X, Wt, L1, L2, 1.0)
    Y2, _ = nf4.lora_forward(X, Wt, L1, L2, 2.0)
    assert np.allclose(Y2 - Y0, 2 * (Y1 - Y0), rtol=0, atol=1e-12)


def test_rel_max_err():
    assert nf4.rel_max_err(np.array([1.0, 2.0]), np.array([1.0, 2.0])) == 0.0
    assert nf4.rel_max_err(np.array([1.1, -4.0]), np.array([1.0, -4.0])) == pytest.approx(0.025)
