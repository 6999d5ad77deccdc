"""The allocation-free forward entry point, checked against the regular one.

qat_linear_fwd_noalloc serves callers that cannot allocate device memory
themselves (a plugin inside a framework that owns all device memory, a
fixed-budget service that allocates only at start-up, latency-critical code
that cannot afford what cudaMalloc / cudaFree may synchronize): its scratch
is a fixed array inside the library.  The test calls it through the C ABI
twice in a row -- with different weights, so the second call must not see
the first call's scratch -- and compares each output with qat_linear_fwd on
the same inputs, within the parity tolerance.  This file sorts last so that
a run stopping at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import synthetic as sy
from parity import assert_close

pytestmark = pytest.mark.gpu


def _regular(W, X, bits, residual=None):
    N, K = W.shape
    Y = torch.empty((X.shape[0], N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(qat.workspace_size(qat.QAT_OP_LINEAR_FWD, N, K, X.shape[0], True),
                     dtype=torch.uint8, device="cuda")
    qat.qat_linear_fwd(X, Y, bits, W=W, residual=residual, workspace=ws)
    return Y


def test_noalloc_matches_regular_forward_twice_in_a_row():
    c1 = sy.linear_case(N=512, K=512, T=256, seed=0)                 # int6 CastedLinear 512->512
    c2 = sy.head_mlp_case(T=333, seed=3)                              # tied head 8192x512 (the maximum)
    cases = [(torch.from_numpy(c1["W"]).cuda(), c1["X"].cuda(), 6),
             (torch.from_numpy(c2["Wemb"]).cuda(), c2["X"].cuda(), 8)]
    for W, X, bits in cases:
        N = W.shape[0]
        Y = torch.empty((X.shape[0], N), dtype=torch.bfloat16, device="cuda")
        qat.qat_linear_fwd_noalloc(W, X, Y, bits)
        ref = _regular(W, X, bits)
        torch.cuda.synchronize()
        assert_close(Y, ref.float().cpu().numpy(), "noalloc vs qat_linear_fwd")
    assert qat.device_error() == 0


def test_noalloc_residual_in_place_and_side_stream():
    """The residual form through the fixed array -- a separate residual, and
    the residual being Y itself (in place) -- on a non-default stream, each
    against qat_linear_fwd on the same inputs."""
    c = sy.linear_case(N=640, K=640, T=1000, seed=4)
    W, X = torch.from_numpy(c["W"]).cuda(), c["X"].cuda()
    R = sy.act_bf16(np.random.default_rng(4), 1000, 640).cuda()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ref = _regular(W, X, 6, residual=R)
        Y = torch.empty_like(R)
        qat.qat_linear_fwd_noalloc(W, X, Y, 6, residual=R, stream=side)
        Yin = R.clone()
        qat.qat_linear_fwd_noalloc(W, X, Yin, 6, residual=Yin, stream=side)
    side.synchronize()
    assert_close(Y, ref.float().cpu().numpy(), "noalloc residual vs qat_linear_fwd")
    assert_close(Yin, ref.float().cpu().numpy(), "noalloc in place vs qat_linear_fwd")
    assert qat.device_error() == 0


def test_noalloc_rejects_weights_beyond_its_scratch():
    L = qat.lib()
    A16 = ctypes.c_void_p(0x10000)
    n = L.qat_linear_fwd_noalloc(A16, 8200, 512, 6, A16, 0, 16, None, A16, None)
    assert n == qat.QAT_ERR_SHAPE
    assert L.qat_linear_fwd_noalloc(A16, 16392, 8, 6, A16, 0, 16, None, A16, None) == qat.QAT_ERR_SHAPE
    # no tokens: nothing to do, as qat_linear_fwd (alignment is not checked then)
    A_BAD = ctypes.c_void_p(0x10004)
    assert L.qat_linear_fwd_noalloc(A_BAD, 512, 512, 6, None, 0, 0, None, None, None) == qat.QAT_OK
    assert L.qat_linear_fwd(A_BAD, None, 512, 512, 6, None, 0, 0, None, None, None, 0, None) == qat.QAT_OK
