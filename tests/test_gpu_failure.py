"""The failure-reporting path of the bounded pipeline waits, exercised on the
GPU without a fault: a probe kernel waits (1 ms) on a barrier that nothing
completes, gives up as a stalled pipeline wait does, and the host reads the
timeout status and the wait site; the context stays usable and the next
regular call is correct."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from _helpers import TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu

OK, ERR_UNSUP, ERR_TIMEOUT = 0, 4, 7
PROBE_TAG_BIT = 1 << 30


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_bounded_wait_gives_up_and_reports_timeout():
    L = q.lib()
    torch.cuda.synchronize()
    assert L.qlora_check_status(_stream()) == OK
    L.qlora_debug_wait_tags()                            # start from a clean record
    assert L.qlora_debug_wait_probe(10, _stream()) == ERR_UNSUP            # limit below 1 us
    assert L.qlora_debug_wait_probe(2_000_000_000, _stream()) == ERR_UNSUP  # limit above 1 s
    assert L.qlora_debug_wait_probe(1_000_000, _stream()) == OK            # 1 ms
    assert L.qlora_check_status(_stream()) == ERR_TIMEOUT
    assert L.qlora_debug_wait_tags() & PROBE_TAG_BIT
    # both records are cleared by reading them
    assert L.qlora_check_status(_stream()) == OK
    assert L.qlora_debug_wait_tags() == 0
    # the context is intact: a regular call afterwards is correct
    layer = Layer(M=16, h=256, o=256, r=8, s=2.0, seed=0)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    Y, _ = q.qlora_linear_fwd(Wq, layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda(), layer.s)
    torch.cuda.synchronize()
    q.qlora_check_status()
    Wb, _ = layer.oracle_weights()
    rY, _ = nf4.lora_forward(layer.f64(layer.X), Wb, layer.f64(layer.L1), layer.f64(layer.L2), layer.s)
    assert nf4.rel_max_err(Y.cpu().numpy().astype(np.float64), rY) <= TOL_SAME_W
