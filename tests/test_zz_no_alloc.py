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
from bit_nf4_quantized_blockwise_b200._lib import QLORA_DTYPE_BF16, QLORA_DTYPE_F32
from _helpers import TOL_BF16_OUT, TOL_SAME_W, Layer

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 8 * 1024 * 1024
ERR_SCRATCH_LIMIT = 9


def _noalloc_via_abi(Wq, X, L1, L2, s, Y, T):
    """Calls the C entry point directly: no workspace, no allocation."""
    st = Wq.struct()
    P = ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)
    dt = QLORA_DTYPE_BF16 if Y.dtype == torch.bfloat16 else QLORA_DTYPE_F32
    return q.lib().qlora_linear_fwd_noalloc(ctypes.byref(st), P(X.data_ptr()), X.shape[0], P(L1.data_ptr()),
                                            P(L2.data_ptr()), L1.shape[1], float(s), P(Y.data_ptr()),
                                            dt, P(T.data_ptr()) if T is not None else None, stream)


def _leave_stale_scratch(h, o, r):
    """A larger no-allocation call on other inputs first, so that the shared
    scratch holds nonzero leftovers when the checked calls run."""
    M = 64
    while q.lib().qlora_linear_fwd_workspace_min_size(o, h, 2 * M, r) <= SCRATCH_LIMIT and M < 1024:
        M *= 2
    other = Layer(M=M, h=h, o=o, r=r, s=1.0, seed=12345)
    Wq = q.quantize_weight(other.W_t.cuda(), other.codebook)
    Y = torch.empty(M, o, dtype=torch.float32, device="cuda")
    T = torch.empty(M, r, dtype=torch.float32, device="cuda")
    assert _noalloc_via_abi(Wq, other.X.cuda(), other.L1.cuda(), other.L2.cuda(), 1.0, Y, T) == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("M,h,o,r,y_dtype", [
    (1, 1024, 640, 64, torch.float32),        # one-token decode
    (2, 1024, 640, 64, torch.bfloat16),       # two tokens, bf16 output (fp32 accumulator in scratch)
    (16, 256, 256, 8, torch.float32),         # decode path, two token groups
    (12, 512, 768, 64, torch.bfloat16),
    (24, 512, 768, 64, torch.float32),        # tensor-memory decode kernel
    (512, 2048, 1536, 64, torch.float32),     # tiled path, several tiles
    (4096, 4096, 4096, 64, torch.float32)])   # a LLaMA-7B-shaped projection (the workspace call
                                              # dequantizes W' into its workspace; this one cannot)
def test_noalloc_matches_workspace_call_twice(M, h, o, r, y_dtype):
    layer = Layer(M=M, h=h, o=o, r=r, s=16.0 / r, seed=M + h + o)
    assert q.lib().qlora_linear_fwd_workspace_min_size(o, h, M, r) <= SCRATCH_LIMIT
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X, L1, L2 = layer.X.cuda(), layer.L1.cuda(), layer.L2.cuda()
    Y_ref, T_ref = q.qlora_linear_fwd(Wq, X, L1, L2, layer.s, y_dtype=y_dtype)
    torch.cuda.synchronize()
    ref_Y = Y_ref.float().cpu().numpy().astype(np.float64)
    ref_T = T_ref.cpu().numpy().astype(np.float64)
    tol = TOL_SAME_W if y_dtype == torch.float32 else TOL_BF16_OUT
    _leave_stale_scratch(h, o, r)
    for call in range(2):
        Y = torch.full((M, o), float("nan"), dtype=y_dtype, device="cuda")
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_via_abi(Wq, X, L1, L2, layer.s, Y, T) == 0
        torch.cuda.synchronize()
        q.qlora_check_status()
        got_Y = Y.float().cpu().numpy().astype(np.float64)
        got_T = T.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got_Y)), call
        assert nf4.rel_max_err(got_Y, ref_Y) <= tol, (call, nf4.rel_max_err(got_Y, ref_Y))
        assert nf4.rel_max_err(got_T, ref_T) <= 1e-5, call


def test_noalloc_rejects_problems_beyond_its_scratch():
    o, h, r = 4096, 4096, 64
    M = 12289  # one token more than fits in 8 MiB at this shape
    assert q.lib().qlora_linear_fwd_workspace_min_size(o, h, M, r) > SCRATCH_LIMIT
    layer = Layer(M=16, h=h, o=o, r=r, s=0.25, seed=1)
    Wq = q.quantize_weight(layer.W_t.cuda(), layer.codebook)
    X = torch.zeros(M, h, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(M, o, dtype=torch.float32, device="cuda")
    before = q.qlora_launch_count()
    rc = _noalloc_via_abi(Wq, X, layer.L1.cuda(), layer.L2.cuda(), 0.25, Y, None)
    assert rc == ERR_SCRATCH_LIMIT
    assert q.qlora_launch_count() == before        # rejected before any launch
    assert not torch.any(Y).item()
