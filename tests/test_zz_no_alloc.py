"""The no-allocation forward entry point (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory at all, such as plug-in
hosts that hand a kernel only its input and output tensors, or runtimes whose
device memory is planned ahead so that nothing may call cudaMalloc during a
step.  Instead of a caller workspace it uses a scratch array compiled into the
library.  Here it is called through the C ABI, twice in a row on the same
inputs, and each result must match the regular qlora_linear_fwd (which takes
a caller workspace) within the tests' tolerance.  The file is named so that
pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import nf4

import bit_nf4_quantized_blockwise_b200 as q
from bit_nf4_quantized_blockwise_b200._lib import QLORA_DTYPE_F32
from _helpers import TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 8 * 1024 * 1024
ERR_SCRATCH_LIMIT = 9


def _noalloc_via_abi(Wq, X, L1, L2, s, Y, T):
    """Calls the C entry point directly: no workspace, no allocation."""
    st = Wq.struct()
    P = ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)
    return q.lib().qlora_linear_fwd_noalloc(ctypes.byref(st), P(X.data_ptr()), X.shape[0], P(L1.data_ptr()),
                                            P(L2.data_ptr()), L1.shape[1], float(s), P(Y.data_ptr()),
                                            QLORA_DTYPE_F32, P(T.data_ptr()) if T is not None else None, stream)


@pytest.mark.parametrize("M,h,o,r", [(16, 256, 256, 8),        # decode path
                                     (512, 2048, 1536, 64),    # tiled path, several tiles
                                     (4096, 4096, 4096, 64)])  # a LLaMA-7B-shaped projection
def test_noalloc_matches_workspace_call_twice(M, h, o, r):
    layer = Layer(M=M, h=h, o=o, r=r, s=16.0 / r, seed=M + h + o)
    assert q.lib().qlora_linear_fwd_workspace_size(o, h, M, r) <= SCRATCH_LIMIT
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, L1, L2 = layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y_ref, T_ref = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s)
    torch.cuda.synchronize()
    ref_Y = Y_ref.cpu().numpy().astype(np.float64)
    ref_T = T_ref.cpu().numpy().astype(np.float64)
    for call in range(2):
        Y = torch.full((M, o), float("nan"), dtype=torch.float32, device="cuda")
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_via_abi(Wq, X, L1, L2, layer.s, Y, T) == 0
        torch.cuda.synchronize()
        q.qlora_check_status()
        got_Y = Y.cpu().numpy().astype(np.float64)
        got_T = T.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got_Y)), call
        assert nf4.rel_max_err(got_Y, ref_Y) <= TOL_SAME_W, (call, nf4.rel_max_err(got_Y, ref_Y))
        assert nf4.rel_max_err(got_T, ref_T) <= 1e-5, call


def test_noalloc_rejects_problems_beyond_its_scratch():
    o, h, r = 4096, 4096, 64
    M = 12289  # one token more than fits in 8 MiB at this shape
    assert q.lib().qlora_linear_fwd_workspace_size(o, h, M, r) > SCRATCH_LIMIT
    layer = Layer(M=16, h=h, o=o, r=r, s=0.25, seed=1)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X = torch.zeros(M, h, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(M, o, dtype=torch.float32, device="cuda")
    before = q.qlora_launch_count()
    rc = _noalloc_via_abi(Wq, X, layer.L1.cuda(), layer.L2.cuda(), 0.25, Y, None)
    assert rc == ERR_SCRATCH_LIMIT
    assert q.qlora_launch_count() == before        # rejected before any launch
    assert not torch.any(Y).item()
