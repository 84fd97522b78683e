"""C-ABI checks that need no GPU: every declared symbol is exported, argument
validation returns the documented status before any launch, and the
quantizer's host-built decision table reproduces the oracle's division rule.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from bit_nf4_quantized_blockwise_b200._lib import qlora_nf4_t

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUP, ERR_CB, ERR_CUDA, ERR_TIMEOUT, ERR_WS = range(9)


@pytest.fixture(scope="module")
def L():
    from bit_nf4_quantized_blockwise_b200 import build
    build.build()
    return q.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
        assert n in q.EXPORTS, n


def test_status_strings_and_version(L):
    assert L.qlora_version() == 10000
    for code in range(9):
        assert L.qlora_status_string(code)
    assert L.qlora_status_string(99) == b"unknown status"


def _cb(values):
    return (ctypes.c_float * 16)(*[float(v) for v in values])


FAKE = 0x10000  # never dereferenced: validation fails before any launch


def test_quantize_validation(L):
    cb = _cb(nf4.nf4_codebook())
    P = ctypes.c_void_p
    assert L.qlora_quantize_nf4(None, 64, ctypes.cast(cb, P), 64, P(FAKE), P(FAKE), None) == ERR_NULL
    assert L.qlora_quantize_nf4(P(FAKE), 64, ctypes.cast(cb, P), 32, P(FAKE), P(FAKE), None) == ERR_UNSUP
    assert L.qlora_quantize_nf4(P(FAKE), 65, ctypes.cast(cb, P), 64, P(FAKE), P(FAKE), None) == ERR_SHAPE
    assert L.qlora_quantize_nf4(P(FAKE), 0, ctypes.cast(cb, P), 64, P(FAKE), P(FAKE), None) == ERR_SHAPE
    assert L.qlora_quantize_nf4(P(FAKE + 2), 64, ctypes.cast(cb, P), 64, P(FAKE), P(FAKE), None) == ERR_ALIGN
    bad = list(nf4.nf4_codebook()); bad[3], bad[4] = bad[4], bad[3]
    assert L.qlora_quantize_nf4(P(FAKE), 64, ctypes.cast(_cb(bad), P), 64, P(FAKE), P(FAKE), None) == ERR_CB
    nozero = list(nf4.nf4_codebook()); nozero[7] = 1e-3
    assert L.qlora_quantize_nf4(P(FAKE), 64, ctypes.cast(_cb(nozero), P), 64, P(FAKE), P(FAKE), None) == ERR_CB
    nan = list(nf4.nf4_codebook()); nan[15] = float("nan")
    assert L.qlora_quantize_nf4(P(FAKE), 64, ctypes.cast(_cb(nan), P), 64, P(FAKE), P(FAKE), None) == ERR_CB


def test_double_quant_validation(L):
    P = ctypes.c_void_p
    ws = L.qlora_double_quant_workspace_size(256, 256)
    assert ws >= 8
    assert L.qlora_double_quant(None, 256, 256, P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws, None) == ERR_NULL
    assert L.qlora_double_quant(P(FAKE), 256, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws, None) == ERR_UNSUP
    assert L.qlora_double_quant(P(FAKE), 300, 256, P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws, None) == ERR_SHAPE
    assert L.qlora_double_quant(P(FAKE), 256, 256, P(FAKE), P(FAKE), P(FAKE), None, ws, None) == ERR_WS
    assert L.qlora_double_quant(P(FAKE), 256, 256, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 4, None) == ERR_WS
    assert L.qlora_double_quant(P(FAKE + 4), 256, 256, P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws, None) == ERR_ALIGN


def _wq(o=256, h=256, block=64, dq_block=256, codebook=None, absmax=None):
    s = qlora_nf4_t()
    s.codes = s.absmax_fp8 = s.dq_scale = s.dq_mean = FAKE
    s.o, s.h = o, h
    s.codebook = _cb(nf4.nf4_codebook() if codebook is None else codebook)
    s.block, s.dq_block = block, dq_block
    if absmax is not None:  # single-level constants: the DQ arrays are unused
        s.absmax = absmax
        s.absmax_fp8 = s.dq_scale = s.dq_mean = None
        s.dq_block = 0
    return s


def test_dequant_and_linear_validation(L):
    P = ctypes.c_void_p
    by = ctypes.byref
    assert L.qlora_dequant(None, P(FAKE), None) == ERR_NULL
    assert L.qlora_dequant(by(_wq(block=32)), P(FAKE), None) == ERR_UNSUP
    assert L.qlora_dequant(by(_wq(o=3, h=64)), P(FAKE), None) == ERR_SHAPE
    assert L.qlora_dequant(by(_wq(h=100)), P(FAKE), None) == ERR_SHAPE
    assert L.qlora_dequant(by(_wq()), None, None) == ERR_NULL
    assert L.qlora_dequant(by(_wq()), P(FAKE + 8), None) == ERR_ALIGN
    w = _wq()
    wsf = L.qlora_linear_fwd_workspace_size(256, 256, 16, 8)
    wsb = L.qlora_linear_bwd_workspace_size(256, 256, 16, 8)
    assert wsb > 0 and wsf > 0
    f = L.qlora_linear_fwd
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 4, 2.0, P(FAKE), 0, None, P(FAKE), wsf, None) == ERR_UNSUP
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 12, 2.0, P(FAKE), 0, None, P(FAKE), wsf, None) == ERR_UNSUP
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 264, 2.0, P(FAKE), 0, None, P(FAKE), wsf, None) == ERR_UNSUP
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 7, None, P(FAKE), wsf, None) == ERR_UNSUP
    assert f(by(w), P(FAKE), 0, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf, None) == ERR_SHAPE
    assert f(by(w), None, 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf, None) == ERR_NULL
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf - 1, None) == ERR_WS
    assert f(by(w), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, P(FAKE + 4), P(FAKE), wsf, None) == ERR_ALIGN
    assert f(by(_wq(o=64, h=64)), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf,
             None) == ERR_SHAPE  # o*h not a whole number of DQ groups
    b = L.qlora_linear_bwd
    args = [P(FAKE), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, None, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), wsb, None]
    assert b(by(w), *args[:-2], wsb - 1, None) == ERR_WS
    bad = list(args); bad[7] = P(FAKE + 4)
    assert b(by(w), *bad) == ERR_ALIGN
    bad = list(args); bad[10] = None
    assert b(by(w), *bad) == ERR_NULL
    assert b(by(_wq(codebook=[0.0] * 16)), *args) == ERR_CB


def test_single_level_constant_validation(L):
    P = ctypes.c_void_p
    by = ctypes.byref
    # double-quantized weights need their three DQ arrays
    w = _wq()
    w.dq_mean = None
    assert L.qlora_dequant(by(w), P(FAKE), None) == ERR_NULL
    # with fp32 block constants they are not needed, nor whole DQ groups:
    # o*h = 64 * 192 is rejected only for the misaligned output, not its shape
    assert L.qlora_dequant(by(_wq(o=64, h=192, absmax=FAKE)), P(FAKE + 8), None) == ERR_ALIGN
    assert L.qlora_dequant(by(_wq(o=64, h=192)), P(FAKE + 8), None) == ERR_SHAPE
    assert L.qlora_dequant(by(_wq(absmax=FAKE + 4)), P(FAKE), None) == ERR_ALIGN
    wsf = L.qlora_linear_fwd_workspace_size(256, 256, 16, 8)
    f = L.qlora_linear_fwd
    assert f(by(_wq(absmax=FAKE)), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf - 1,
             None) == ERR_WS
    assert f(by(_wq(absmax=FAKE + 4)), P(FAKE), 16, P(FAKE), P(FAKE), 8, 2.0, P(FAKE), 0, None, P(FAKE), wsf,
             None) == ERR_ALIGN


# ---------------------------------------------------------------- decision table

def _all_bf16_in(c_bits):
    """Every bf16 bit pattern with |value| <= the value of c_bits (positive)."""
    mags = np.arange(0, c_bits + 1, dtype=np.uint16)
    return np.concatenate([mags, mags | np.uint16(0x8000)])


def _table_codes(w_bits, table_row, k):
    """code = #{j : w > B_j * 2^k}, the rule the quantize kernel applies."""
    b = table_row[:15].astype(np.int64) + (k << 7)
    bv = nf4.bf16_bits_to_f32(b.astype(np.uint16))
    wv = nf4.bf16_bits_to_f32(w_bits)
    return np.sum(wv[:, None] > bv[None, :], axis=1)


@pytest.mark.parametrize("name", ["nf4", "uniform", "fp4_e2m1"])
def test_decision_table_matches_division_rule(name):
    if name == "nf4":
        cb = nf4.nf4_codebook()
    elif name == "uniform":
        cb = ((np.arange(16) - 7) / 8.0).astype(np.float32)
    else:  # FP4 E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, normalised, one zero
        m = np.array([0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
        cb = np.concatenate([-m[::-1][:7], [0.0], m, [8.0]])[:16] / 8.0
        cb = np.sort(cb).astype(np.float32)
    nf4.validate_codebook(cb)
    tab = q.qlora_nf4_boundaries(cb)
    t = nf4.nearest_code_thresholds(cb)
    for m in range(128):
        cbits = (127 << 7) | m
        c = nf4.bf16_bits_to_f32(np.array([cbits], np.uint16))[0]
        w = _all_bf16_in(cbits)
        x = (nf4.bf16_bits_to_f32(w) / c).astype(np.float32)
        ref = np.sum(x[:, None] > t[None, :], axis=1)
        got = _table_codes(w, tab[m], 0)
        assert np.array_equal(got, ref), (name, m)
        assert np.all(np.diff(nf4.bf16_bits_to_f32(tab[m][:15])) >= 0)


def test_decision_table_scales_with_the_absmax_exponent():
    # Blocks whose absmax spans 2^-100 .. 2^100: the exponent-shifted table
    # gives the oracle's codes for every element.
    cb = nf4.nf4_codebook()
    tab = q.qlora_nf4_boundaries(cb)
    rng = np.random.default_rng(0)
    for k in (-100, -37, -8, -1, 0, 1, 5, 60, 100):
        vals = rng.standard_normal(64 * 64) * 2.0 ** k
        w = nf4.f32_to_bf16_bits(vals.astype(np.float32))
        codes, absmax = nf4.quantize_blockwise(w, cb)
        for b in range(64):
            cbits = int(nf4.f32_to_bf16_bits(absmax[b:b + 1])[0])
            kk = (cbits >> 7) - 127
            got = _table_codes(w[b * 64:(b + 1) * 64], tab[cbits & 0x7F], kk)
            assert np.array_equal(got, codes[b * 64:(b + 1) * 64]), (k, b)


def _bins(w_bits):
    """The quantize kernel's bin of a scaled element: bf16(31 x + 192) - 128
    (31 x + 192 is exact in double; numpy's rint rounds to nearest even)."""
    return (np.rint(31.0 * nf4.bf16_bits_to_f32(w_bits).astype(np.float64) + 192.0) - 128).astype(np.int64)


def _bin_row(row):
    """The kernel's (bin -> {base, thr}) row for one significand: base = number of
    boundaries in lower bins; thr = the bin's boundary when an element of the
    bin can exceed it (its bf16 successor has the same bin), else +inf."""
    b = row[:15].astype(np.uint16)
    bin_b = _bins(b)
    succ = np.where(b & 0x8000, b - 1, b + 1).astype(np.uint16)
    exceedable = _bins(succ) == bin_b
    base = np.array([np.sum(bin_b < k) for k in range(128)])
    thr = np.full(128, np.inf)
    for j in range(15):
        if exceedable[j]:
            thr[bin_b[j]] = nf4.bf16_bits_to_f32(b[j:j + 1])[0]
    return bin_b, base, thr


@pytest.mark.parametrize("name", ["nf4", "uniform", "fp4_e2m1"])
def test_bin_lookup_matches_division_rule(name):
    # The bin-table path of the quantize kernel, restated here from its
    # definition: for every significand row and every bf16 element within the
    # absmax, base(bin) + [x > thr(bin)] must equal the oracle's division rule.
    if name == "nf4":
        cb = nf4.nf4_codebook()
    elif name == "uniform":
        cb = ((np.arange(16) - 7) / 8.0).astype(np.float32)
    else:
        m = np.array([0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
        cb = np.sort(np.concatenate([-m[::-1][:7], [0.0], m, [8.0]])[:16] / 8.0).astype(np.float32)
    tab = q.qlora_nf4_boundaries(cb)
    t = nf4.nearest_code_thresholds(cb)
    for m in range(128):
        bin_b, base, thr = _bin_row(tab[m])
        assert np.all(np.diff(bin_b) > 0), (name, m)  # the path's precondition holds for these codebooks
        cbits = (127 << 7) | m
        c = nf4.bf16_bits_to_f32(np.array([cbits], np.uint16))[0]
        w = _all_bf16_in(cbits)
        x = (nf4.bf16_bits_to_f32(w) / c).astype(np.float32)
        ref = np.sum(x[:, None] > t[None, :], axis=1)
        k = _bins(w)
        assert k.min() >= 2 and k.max() <= 126
        got = base[k] + (nf4.bf16_bits_to_f32(w) > thr[k])
        assert np.array_equal(got, ref), (name, m)


def test_library_codebook_matches_oracle_bit_exact(L):
    lib_cb = np.array(q.qlora_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(lib_cb.view(np.uint32), nf4.nf4_codebook().view(np.uint32))


def test_workspace_sizes_of_the_two_weight_product_paths(L):
    # Below 1024 tokens the full and the minimum workspace coincide (the fused
    # dequant-GEMM runs).  From 1024 tokens the full size adds the bf16 W'
    # (o*h*2 bytes) and the split-tail buffers of the SM-pair GEMM, and a call
    # given only the minimum still runs (on the fused kernel): the minimum is
    # what a call must receive, the full size what selects the faster path.
    o, h, r = 4096, 11008, 64
    for M in (16, 512, 1023):
        assert L.qlora_linear_fwd_workspace_size(o, h, M, r) == L.qlora_linear_fwd_workspace_min_size(o, h, M, r)
        assert L.qlora_linear_bwd_workspace_size(o, h, M, r) == L.qlora_linear_bwd_workspace_min_size(o, h, M, r)
    for M in (1024, 4096):
        for full, small in ((L.qlora_linear_fwd_workspace_size, L.qlora_linear_fwd_workspace_min_size),
                            (L.qlora_linear_bwd_workspace_size, L.qlora_linear_bwd_workspace_min_size),
                            (L.qlora_linear_fwd_dropout_workspace_size, L.qlora_linear_fwd_dropout_workspace_min_size),
                            (L.qlora_linear_bwd_dropout_workspace_size, L.qlora_linear_bwd_dropout_workspace_min_size)):
            extra = full(o, h, M, r) - small(o, h, M, r)
            assert extra >= o * h * 2, (M, extra)
            assert extra < o * h * 2 + 64 * 1024 * 1024, (M, extra)  # W' plus the tail buffers (< 64 MiB)
    # the minimum does not grow with the weight-product path: it stays far below W'
    assert L.qlora_linear_fwd_workspace_min_size(o, h, 4096, r) < o * h * 2
