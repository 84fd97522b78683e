"""Data-parallel path on CPU: two gloo ranks each run the layer's backward on
their own tokens (the oracle stands in for the kernels), exchange the LoRA
gradients with the same helper bench.py uses, and must obtain the gradient of
the full batch.  No GPU is involved."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_blockwise_b200 import dp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    import synth
    M, h, o, r, s = 24, 128, 192, 8, 2.0
    X = synth.activations(M, h, seed=3).double().numpy()
    dY = synth.activations(M, o, seed=3, tag="dY").double().numpy()
    Wt = synth.weight_t(o, h, seed=3).double().numpy()
    L1, L2 = (t.double().numpy() for t in synth.lora_factors(h, r, o, seed=3))
    return M, h, o, r, s, X, dY, Wt, L1, L2


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import nf4
        M, h, o, r, s, X, dY, Wt, L1, L2 = _layer()
        b, e = dp.shard_rows(M, rank, world)
        _, dL1, dL2, _, _ = nf4.lora_backward(X[b:e], dY[b:e], Wt, L1, L2, s)
        flat, g1, g2 = dp.lora_grad_buffers(h, o, r, "cpu", dtype=torch.float64)
        g1.copy_(torch.from_numpy(dL1))
        g2.copy_(torch.from_numpy(dL2))
        dp.allreduce_lora_grads(flat)
        q.put((rank, g1.numpy().copy(), g2.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_the_batch():
    for M in (1, 7, 24, 4096):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(M, k, world) for k in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(spans[k][1] == spans[k + 1][0] for k in range(world - 1))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1


def test_allreduce_is_noop_without_process_group():
    flat, g1, g2 = dp.lora_grad_buffers(4, 6, 2, "cpu")
    flat.fill_(1.5)
    dp.allreduce_lora_grads(flat)
    assert torch.all(flat == 1.5) and g1.shape == (4, 2) and g2.shape == (2, 6)


@pytest.mark.timeout(300)
def test_two_rank_gradient_exchange_equals_full_batch():
    from oracle import nf4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(k, 2, port, q)) for k in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    M, h, o, r, s, X, dY, Wt, L1, L2 = _layer()
    _, rdL1, rdL2, _, _ = nf4.lora_backward(X, dY, Wt, L1, L2, s)
    for _, g1, g2 in got:
        assert np.allclose(g1, rdL1, rtol=1e-12, atol=1e-14)
        assert np.allclose(g2, rdL2, rtol=1e-12, atol=1e-14)
