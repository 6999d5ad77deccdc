"""GPU parity of the QAT linear (tcgen05 GEMM with the quantized operand)
against the fp64 oracle: forward, residual and strided-input forms, STE
backward dX / dW, and dW accumulation over recurrent uses."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import synthetic as sy
from parity import assert_close

pytestmark = pytest.mark.gpu


def _x(t):
    return t.float().numpy()


@pytest.mark.parametrize("raw", [True, False])
def test_linear_fwd_cfg1(raw):
    """Single int6 CastedLinear 512->512, T=256 (one M tile, two N tiles)."""
    c = sy.linear_case()
    W, X = c["W"], c["X"]
    Wd, Xd = torch.from_numpy(W).cuda(), X.cuda()
    Y = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
    if raw:
        ws = torch.empty(qat.workspace_size(qat.QAT_OP_LINEAR_FWD, 512, 512, 256, True),
                         dtype=torch.uint8, device="cuda")
        qat.qat_linear_fwd(Xd, Y, 6, W=Wd, workspace=ws)
    else:
        qat.qat_linear_fwd(Xd, Y, 6, qw=qat.quantize_weight(Wd, 6))
    torch.cuda.synchronize()
    ref = o.linear_fwd(o.quantize_weight(W, 6)["operand"], _x(X))
    assert_close(Y, ref, "Y")
    assert qat.device_error() == 0


@pytest.mark.parametrize("shape", [(333, 136, 200), (1, 8, 8), (129, 264, 72), (700, 512, 1536),
                                   (600, 200, 136), (520, 264, 512), (1024, 640, 640)])
@pytest.mark.parametrize("bits", [6, 8])
def test_linear_fwd_ragged_and_residual(shape, bits):
    """Ragged T (M tail), N not a multiple of the tile, K not a multiple of 64;
    with at least 256 rows the forward runs on CTA pairs 256 columns wide, so
    N = 200, 264 (a second block of 8 columns) and 640 end in a partial block."""
    T, N, K = shape
    rng = np.random.default_rng(T + N + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    X = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float32)).to(torch.bfloat16)
    Rs = torch.from_numpy(rng.standard_normal((T, N)).astype(np.float32)).to(torch.bfloat16)
    q = qat.quantize_weight(torch.from_numpy(W).cuda(), bits)
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    Rd = Rs.cuda()
    qat.qat_linear_fwd(X.cuda(), Y, bits, qw=q)
    Y2 = Rd.clone()
    qat.qat_linear_fwd(X.cuda(), Y2, bits, qw=q, residual=Y2)  # in place: Y aliases residual
    torch.cuda.synchronize()
    op = o.quantize_weight(W, bits)["operand"]
    ref = o.linear_fwd(op, _x(X))
    assert_close(Y, ref, "Y")
    assert_close(Y2, ref + _x(Rs), "Y+residual")


def test_linear_fwd_strided_input():
    """X read through a row stride (the query slice of a fused QKV output)."""
    rng = np.random.default_rng(3)
    T, K, ld, N = 300, 640, 1280, 640
    big = torch.from_numpy(rng.standard_normal((T, ld)).astype(np.float32)).to(torch.bfloat16)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    q = qat.quantize_weight(torch.from_numpy(W).cuda(), 6)
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    qat.qat_linear_fwd(big.cuda(), Y, 6, qw=q, ldx=ld, T=T)
    torch.cuda.synchronize()
    assert_close(Y, o.linear_fwd(o.quantize_weight(W, 6)["operand"], _x(big)[:, :K]), "Y")


@pytest.mark.parametrize("shape", [(333, 136, 200), (256, 512, 512), (2000, 264, 72)])
def test_linear_bwd_and_dw_accumulation(shape):
    T, N, K = shape
    rng = np.random.default_rng(T * 7 + N)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Xs = [torch.from_numpy(rng.standard_normal((T, K)).astype(np.float32)).to(torch.bfloat16) for _ in range(3)]
    dYs = [torch.from_numpy((rng.standard_normal((T, N)) * 0.01).astype(np.float32)).to(torch.bfloat16) for _ in range(3)]
    Wd = torch.from_numpy(W).cuda()
    ws = torch.empty(qat.workspace_size(qat.QAT_OP_LINEAR_BWD, N, K, T, True), dtype=torch.uint8, device="cuda")
    dX = torch.empty((T, K), dtype=torch.bfloat16, device="cuda")
    dW = torch.full((N, K), 7.0, dtype=torch.float32, device="cuda")
    qat.qat_linear_bwd(Xs[0].cuda(), dYs[0].cuda(), 6, W=Wd, dX=dX, dW=dW, workspace=ws)
    torch.cuda.synchronize()
    op = o.quantize_weight(W, 6)["operand"]
    rdX, rdW = o.linear_bwd(op, _x(Xs[0]), _x(dYs[0]))
    assert_close(dX, rdX, "dX")
    assert_close(dW, rdW, "dW")
    # R = 3 recurrent uses: gradients accumulate into dW
    for i in (1, 2):
        qat.qat_linear_bwd(Xs[i].cuda(), dYs[i].cuda(), 6, qw=None, W=None, dW=dW,
                           accumulate_dW=True, N=N, K=K)
    torch.cuda.synchronize()
    tot = sum(o.linear_bwd(op, _x(x), _x(g))[1] for x, g in zip(Xs, dYs))
    assert_close(dW, tot, "dW accumulated over 3 uses")
    assert qat.device_error() == 0


@pytest.mark.parametrize("shape", [(333, 136, 200), (1000, 640, 640), (4096, 640, 640)])
@pytest.mark.parametrize("alias", [False, True])
def test_linear_bwd_strided_input_and_dx_residual(shape, alias):
    """The backward given X as a column slice of a wider activation (row
    stride ldx) and a dX residual, added before the bf16 rounding -- also
    when the residual is dX itself (in place)."""
    T, N, K = shape
    rng = np.random.default_rng(T + N + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    wide = torch.from_numpy(rng.standard_normal((T, 2 * K + 8)).astype(np.float32)).to(torch.bfloat16)
    X = wide[:, 8:8 + K]
    dY = torch.from_numpy((rng.standard_normal((T, N)) * 0.01).astype(np.float32)).to(torch.bfloat16)
    Rs = torch.from_numpy((rng.standard_normal((T, K)) * 0.01).astype(np.float32)).to(torch.bfloat16)
    q = qat.quantize_weight(torch.from_numpy(W).cuda(), 6)
    wd = wide.cuda()
    Rd = Rs.cuda()
    dX = Rd if alias else torch.empty((T, K), dtype=torch.bfloat16, device="cuda")
    dW = torch.empty((N, K), dtype=torch.float32, device="cuda")
    qat.qat_linear_bwd(wd[:, 8:], dY.cuda(), 6, qw=q, dX=dX, dW=dW, ldx=2 * K + 8, dX_residual=Rd)
    torch.cuda.synchronize()
    op = o.quantize_weight(W, 6)["operand"]
    rdX, rdW = o.linear_bwd(op, _x(X), _x(dY))
    assert_close(dX, rdX + _x(Rs), "dX + residual")
    assert_close(dW, rdW, "dW from the strided X")
    assert qat.device_error() == 0


def test_zero_tokens_is_a_noop():
    q = qat.quantize_weight(torch.zeros((64, 64), device="cuda"), 6)
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    qat.qat_linear_fwd(X, Y, 6, qw=q)
    dW = torch.full((64, 64), 3.0, device="cuda")
    qat.qat_linear_bwd(X, Y, 6, dW=dW, N=64, K=64)
    torch.cuda.synchronize()
    assert torch.all(dW == 0)
