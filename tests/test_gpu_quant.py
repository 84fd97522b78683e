"""GPU parity of NF4 quantization, double quantization and dequantization
against the CPU oracle: codes, absmax, FP8 constants, dq_scale, dq_mean and
the dequantized bf16 weight must match bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import OTHER_CODEBOOKS, bits, oracle_quantized

pytestmark = pytest.mark.gpu

CODEBOOKS = {
    "nf4": nf4.nf4_codebook(),
    "uniform": ((np.arange(16) - 7) / 8.0).astype(np.float32),
    "fp4_e2m1": np.sort(np.concatenate([-np.array([6, 4, 3, 2, 1.5, 1, 0.5]), [0.0],
                                        [0.5, 1, 1.5, 2, 3, 4, 6, 8]]) / 8.0).astype(np.float32),
    # Codebooks outside the range the f16 counting path accepts (boundaries in
    # [2^-6, 2) in magnitude): values up to 3, values 1e-3 next to zero, and a
    # subnormal value, which send the quantizer down its other two paths.
    "nf4_x3": (nf4.nf4_codebook().astype(np.float64) * 3).astype(np.float32),
    "tiny_center": np.where(np.abs(nf4.nf4_codebook()) < 0.1,
                            np.sign(nf4.nf4_codebook()) * 1e-3, nf4.nf4_codebook()).astype(np.float32),
    "subnormal": np.where(np.arange(16) == 8, np.float32(2e-39), nf4.nf4_codebook()).astype(np.float32),
    "fp4_e3m0": OTHER_CODEBOOKS["fp4_e3m0"],
}


def _gpu_quantize(w_t, codebook):
    codes, absmax = q.qlora_quantize_nf4(w_t.cuda(), codebook)
    torch.cuda.synchronize()
    q.qlora_check_status()
    return codes.cpu().numpy(), absmax.cpu().numpy()


@pytest.mark.parametrize("shape", [(256, 256), (64, 64), (3, 64 * 5), (1, 64), (129, 192), (1000, 1088)])
@pytest.mark.parametrize("cb", list(CODEBOOKS))
def test_quantize_bit_exact(shape, cb):
    o, h = shape
    w = synth.weight_t(o, h, seed=o * 7 + h, outlier_frac=0.001 if o * h > 10000 else 0.0)
    codes, absmax = _gpu_quantize(w, CODEBOOKS[cb])
    ref_codes, ref_absmax = nf4.quantize_blockwise(bits(w), CODEBOOKS[cb])
    assert np.array_equal(absmax.view(np.uint32), ref_absmax.view(np.uint32))
    assert np.array_equal(codes, nf4.pack_codes(ref_codes))


def test_quantize_edge_blocks():
    # all-zero (both signs), codebook-valued, absmax-only, subnormal and huge
    # scales, exact threshold ties (uniform codebook), and an alternating pattern.
    rng = np.random.default_rng(1)
    blocks = [np.zeros(64), -np.zeros(64)]
    for c in (1.0, 0.037, 2.0 ** -130, 2.0 ** -126, 1e-38, 3e38, 2.0 ** 120, 1e-20):
        blocks.append(rng.uniform(-c, c, 64))
        v = np.concatenate([nf4.nf4_codebook() * c, rng.uniform(-c, c, 48)])
        blocks.append(v)
    blocks.append(np.where(np.arange(64) % 2 == 0, 1.0, -1.0) * 0.25)
    t = nf4.nearest_code_thresholds(CODEBOOKS["uniform"])
    blocks.append(np.concatenate([[1.0], t, -t, rng.uniform(-1, 1, 64 - 31)]))
    for cb in CODEBOOKS.values():
        blocks.append(np.concatenate([[1.0], nf4.nearest_code_thresholds(cb), rng.uniform(-1, 1, 48)]))
    w = np.concatenate(blocks).astype(np.float32)
    wb = nf4.f32_to_bf16_bits(w)
    for name, cb in CODEBOOKS.items():
        codes, absmax = _gpu_quantize(torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16), cb)
        ref_codes, ref_absmax = nf4.quantize_blockwise(wb, cb)
        assert np.array_equal(absmax.view(np.uint32), ref_absmax.view(np.uint32)), name
        assert np.array_equal(codes, nf4.pack_codes(ref_codes)), name


def _random_codebook(rng, min_gap):
    """16 strictly increasing values in [-1, 1], exactly one 0.0, the largest
    magnitude 1, neighbouring values at least min_gap apart."""
    while True:
        neg = -np.sort(rng.uniform(min_gap, 1.0, 7))[::-1]
        pos = np.sort(rng.uniform(min_gap, 1.0, 8))
        v = np.concatenate([neg, [0.0], pos])
        v = v / np.max(np.abs(v))
        v32 = v.astype(np.float32)
        if np.all(np.diff(v32.astype(np.float64)) >= min_gap) and np.count_nonzero(v32 == 0) == 1:
            return v32


@pytest.mark.parametrize("trial", range(6))
def test_quantize_random_codebooks_every_significand(trial):
    # Random codebooks (wide gaps, which the quantizer's bin lookup serves, and
    # narrow ones, which send it to its search), on blocks whose absmax runs
    # through all 128 bf16 significands at binades 2^-40 .. 2^40.
    rng = np.random.default_rng(100 + trial)
    cb = _random_codebook(rng, 0.09 if trial % 2 == 0 else 0.01)
    nb = 128 * 9
    w = rng.standard_normal((nb, 64))
    w /= np.max(np.abs(w), axis=1, keepdims=True)
    sig = 1.0 + (np.arange(nb) % 128) / 128.0
    e = 2.0 ** (10 * ((np.arange(nb) // 128) - 4))
    w *= (sig * e)[:, None]
    w[np.arange(nb), rng.integers(0, 64, nb)] = sig * e * np.where(np.arange(nb) % 3 == 0, -1.0, 1.0)
    wb = nf4.f32_to_bf16_bits(w.reshape(-1).astype(np.float32))
    codes, absmax = _gpu_quantize(torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16), cb)
    ref_codes, ref_absmax = nf4.quantize_blockwise(wb, cb)
    assert np.array_equal(absmax.view(np.uint32), ref_absmax.view(np.uint32))
    assert np.array_equal(codes, nf4.pack_codes(ref_codes))


@pytest.mark.parametrize("nb", [256, 512, 256 * 37])
def test_double_quant_bit_exact(nb):
    rng = np.random.default_rng(nb)
    c = nf4.bf16_bits_to_f32(nf4.f32_to_bf16_bits(np.abs(rng.standard_normal(nb) * 0.02).astype(np.float32)))
    c[5] = 0.0                        # an all-zero block
    if nb >= 512:
        c[256:512] = c[300]           # a group with dq_scale = 0 only if it equals the mean; keep generic
    a = torch.from_numpy(c).cuda()
    e, sc, mu = q.qlora_double_quant(a)
    torch.cuda.synchronize()
    re, rsc, rmu = nf4.double_quant(c)
    assert mu.cpu().numpy().view(np.uint32)[0] == np.float32(rmu).view(np.uint32)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
    assert np.array_equal(e.cpu().numpy(), re)


def test_double_quant_constant_group_and_saturation():
    # Every constant equal: mean exact, dq_scale 0, codes 0.  Two-valued groups
    # map to exactly -448 / +448.
    c = np.full(512, 0.0625, np.float32)
    e, sc, mu = q.qlora_double_quant(torch.from_numpy(c).cuda())
    assert float(mu.item()) == 0.0625 and not sc.cpu().numpy().any() and not e.cpu().numpy().any()
    c = np.array([0.0234375, 0.0390625] * 256, np.float32)
    e, sc, mu = q.qlora_double_quant(torch.from_numpy(c).cuda())
    re, rsc, rmu = nf4.double_quant(c)
    assert np.array_equal(e.cpu().numpy(), re) and set(re.tolist()) == {0x7E, 0xFE}


@pytest.mark.parametrize("shape", [(256, 256), (512, 320), (4096, 4096)])
def test_quantize_dq_dequant_pipeline_bit_exact(shape):
    o, h = shape
    w = synth.weight_t(o, h, seed=3, outlier_frac=0.001)
    cb = nf4.nf4_codebook()
    Wq = q.quantize_weight(w.cuda(), cb)
    Wd = q.qlora_dequant(Wq)
    torch.cuda.synchronize()
    q.qlora_check_status()
    cp, absmax, e, sc, mu = oracle_quantized(w, cb)
    assert np.array_equal(Wq.codes.cpu().numpy(), cp)
    assert np.array_equal(Wq.absmax_fp8.cpu().numpy(), e)
    assert np.array_equal(Wq.dq_scale.cpu().numpy().view(np.uint32), sc.view(np.uint32))
    assert Wq.dq_mean.cpu().numpy().view(np.uint32)[0] == np.float32(mu).view(np.uint32)
    ref = nf4.dequant(cp, e, sc, mu, cb)
    assert np.array_equal(bits(Wd), ref)


def test_dequant_of_oracle_constants_bit_exact():
    # The dequant kernel fed the oracle's own quantized tuple (independent of
    # the GPU quantizer), with a second codebook.
    o, h = 192, 256
    cb = CODEBOOKS["fp4_e2m1"]
    w = synth.weight_t(o, h, seed=9)
    cp, absmax, e, sc, mu = oracle_quantized(w, cb)
    Wq = q.NF4Weight(torch.from_numpy(cp).cuda(), torch.from_numpy(e).cuda(), torch.from_numpy(sc).cuda(),
                     torch.tensor([mu], dtype=torch.float32).cuda(), o, h, tuple(float(v) for v in cb))
    Wd = q.qlora_dequant(Wq)
    torch.cuda.synchronize()
    assert np.array_equal(bits(Wd), nf4.dequant(cp, e, sc, mu, cb))
