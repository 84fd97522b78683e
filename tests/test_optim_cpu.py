"""CPU checks of the LoRA optimizer: the oracle AdamW against torch's AdamW
and gradient clipping (fp64), its closed-form first step, and the paged
optimizer's host-side policy against a fake memory probe (no GPU)."""
import math

import numpy as np
import torch

from oracle import optim

from bit_nf4_quantized_blockwise_b200.paged import PagingPolicy


def test_oracle_adamw_matches_torch_adamw_with_clipping():
    rng = np.random.default_rng(0)
    shapes = [(64, 8), (8, 48), (33,)]
    cfg = dict(lr=2e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    P = [rng.standard_normal(s) * 0.05 for s in shapes]
    tp = [torch.tensor(p, dtype=torch.float64, requires_grad=True) for p in P]
    opt = torch.optim.AdamW(tp, lr=cfg["lr"], betas=(cfg["beta1"], cfg["beta2"]), eps=cfg["eps"],
                            weight_decay=cfg["weight_decay"], foreach=False)
    op = [p.copy() for p in P]
    m = [np.zeros_like(p) for p in P]
    v = [np.zeros_like(p) for p in P]
    for t in range(1, 7):
        grads = [rng.standard_normal(s) * (0.3 if t % 2 else 3.0) for s in shapes]  # clipping active on even steps
        for p, g in zip(tp, grads):
            p.grad = torch.tensor(g, dtype=torch.float64)
        torch.nn.utils.clip_grad_norm_(tp, 0.3)
        opt.step()
        optim.adamw_step(op, grads, m, v, t, max_grad_norm=0.3, **cfg)
        for a, b in zip(op, tp):
            assert np.max(np.abs(a - b.detach().numpy())) <= 1e-14
        for mi, vi, b in zip(m, v, tp):
            st = opt.state[b]
            assert np.max(np.abs(mi - st["exp_avg"].numpy())) <= 1e-15
            assert np.max(np.abs(vi - st["exp_avg_sq"].numpy())) <= 1e-15


def test_oracle_adamw_first_step_closed_form():
    # t = 1, no decay, no clipping: m^ = g and sqrt(v^) = |g|, so p1 = p0 - lr g / (|g| + eps)
    g = np.array([0.5, -2.0, 1e-3, 0.0])
    p = [np.array([1.0, 1.0, 1.0, 1.0])]
    optim.adamw_step(p, [g], [np.zeros(4)], [np.zeros(4)], 1, lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8,
                     weight_decay=0.0, max_grad_norm=None)
    assert np.allclose(p[0], 1.0 - 0.1 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-15)
    assert math.isclose(optim.clip_coefficient([np.array([3.0, 4.0])], 0.3), 0.3 / (5.0 + 1e-6))
    assert optim.clip_coefficient([np.array([0.1, 0.1])], 0.3) == 1.0


def test_paging_policy_moves_state_under_pressure_and_back():
    free = {"v": 10_000}
    moved = []
    pol = PagingPolicy(state_bytes=3_000, watermark=2_000, mem_info=lambda: (free["v"], 20_000),
                       move=lambda to_host: moved.append(to_host))
    assert not pol.on_pressure() and not pol.on_host        # plenty free: stays on the device
    free["v"] = 1_500                                        # a spike
    assert pol.on_pressure() and pol.on_host and moved == [True]
    assert not pol.on_pressure()                              # already on the host
    free["v"] = 4_000                                         # 4000 - 3000 < 2000: no room to bring it back
    assert not pol.on_step() and pol.on_host
    free["v"] = 6_000                                         # 6000 - 3000 >= 2000
    assert pol.on_step() and not pol.on_host and moved == [True, False]
    assert pol.moves == ["to_host", "to_device"]
    assert not pol.on_step()
