"""GPU parity of the paged AdamW step of the LoRA factors against the fp64
oracle, with the optimizer state in unified memory: resident, evicted to host
RAM between steps (what a memory spike does), and moved by the paging policy
under a (fake) memory-pressure signal.  Eviction changes where the state
lives, not the arithmetic, so those runs match the resident one bit for bit."""
import numpy as np
import pytest
import torch

from oracle import optim

from bit_nf4_quantized_blockwise_b200.paged import AdamWConfig, PagedAdamW, flat_views

pytestmark = pytest.mark.gpu

SHAPES = [(1024, 64), (64, 640), (512, 16), (16, 1024)]
CFG = AdamWConfig(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, max_grad_norm=0.3)


def _grads(step):
    g = torch.Generator().manual_seed(100 + step)
    scale = 0.002 if step % 2 else 0.05   # clipping active on even steps
    return [torch.randn(s, generator=g) * scale for s in SHAPES]


def _run(evict_at=(), pressure=None, steps=5):
    g0 = torch.Generator().manual_seed(1)
    n = sum(a * b for a, b in SHAPES)
    param = torch.cat([(torch.randn(s, generator=g0) * 0.01).reshape(-1) for s in SHAPES]).cuda()
    copy = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    kw = {}
    if pressure is not None:
        kw = dict(watermark_bytes=1 << 30, mem_info=pressure)
    opt = PagedAdamW(param, CFG, copy=copy, **kw)
    for t in range(1, steps + 1):
        if t in evict_at:
            opt.evict()
        if pressure is not None:
            opt.policy.on_pressure()
        opt.step(torch.cat([g.reshape(-1) for g in _grads(t)]).cuda())
    torch.cuda.synchronize()
    P = [v.cpu().numpy() for v in flat_views(param, SHAPES)]
    M = [v.cpu().numpy() for v in flat_views(opt.m.tensor, SHAPES)]
    V = [v.cpu().numpy() for v in flat_views(opt.v.tensor, SHAPES)]
    C = [v.cpu() for v in flat_views(copy, SHAPES)]
    out = (P, M, V, C, list(opt.policy.moves))
    opt.close()
    return out


def test_paged_adamw_matches_oracle():
    P, M, V, C, _ = _run()
    g0 = torch.Generator().manual_seed(1)
    op = [(torch.randn(s, generator=g0) * 0.01).double().numpy() for s in SHAPES]
    om = [np.zeros(s) for s in SHAPES]
    ov = [np.zeros(s) for s in SHAPES]
    # the oracle gets the hyper-parameters as the library receives them (fp32 values)
    f32 = lambda x: float(np.float32(x))  # noqa: E731
    for t in range(1, 6):
        optim.adamw_step(op, [g.double().numpy() for g in _grads(t)], om, ov, t, lr=f32(CFG.lr), beta1=f32(CFG.beta1),
                         beta2=f32(CFG.beta2), eps=f32(CFG.eps), weight_decay=f32(CFG.weight_decay),
                         max_grad_norm=f32(CFG.max_grad_norm))
    for a, b in zip(P, op):
        assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(b))
    for a, b in zip(M, om):
        assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(b))
    for a, b in zip(V, ov):
        assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(b))
    for p, c in zip(P, C):   # the bf16 copy the layer reads is the rounding of the fp32 parameter
        assert torch.equal(c, torch.from_numpy(p).to(torch.bfloat16))


def test_evicted_state_gives_identical_steps():
    base = _run()
    ev = _run(evict_at=(2, 4))
    for a, b in zip(base[0] + base[1] + base[2], ev[0] + ev[1] + ev[2]):
        assert np.array_equal(a, b)
    # evicted before steps 2 and 4; with room on the device each step brings it back first
    assert ev[4] == ["to_host", "to_device", "to_host", "to_device"]


def test_memory_pressure_policy_moves_state_and_back():
    # fake probe: a spike (little free memory) before steps 2 and 3, ample memory otherwise
    calls = {"n": 0}

    def probe():
        calls["n"] += 1
        spike = calls["n"] in (3, 4, 5)
        return ((1 << 29) if spike else (1 << 34), 1 << 35)
    base = _run()
    got = _run(pressure=probe)
    for a, b in zip(base[0] + base[1] + base[2], got[0] + got[1] + got[2]):
        assert np.array_equal(a, b)
    assert "to_host" in got[4] and "to_device" in got[4]
