"""GPU parity of the forward GEMMs that quantize their fp32 weight inside the
GEMM (the fused quantizing B producer: row amax, scale, codes and the bf16
STE operand built in shared memory, never written to global memory).

qat_linear_fwd and qat_mlp_fwd take this path when given fp32 weights, no
workspace and at least 256 tokens.  Checked against the fp64 oracle on the quantized operand,
and bit for bit against the same GEMM fed the operand materialised by
qat_quantize_weights where both pick the same tile shape (N a multiple of 256,
K <= 512): the operand bits and the accumulation order are then the same.
The shapes cover every panel width (256, 192, 160 and 128 columns per CTA
pair), ragged N and K, and runs of tiles that cross N blocks (the panel is
rebuilt mid-kernel)."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat
from parity import assert_close, bits16

pytestmark = pytest.mark.gpu


def _case(T, N, K, seed, outliers=True):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    if outliers:  # a few large entries so row scales differ widely
        idx = rng.choice(N * K, size=max(1, N * K // 1000), replace=False)
        W.reshape(-1)[idx] *= 20.0
    X = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float32)).to(torch.bfloat16)
    R = torch.from_numpy(rng.standard_normal((T, N)).astype(np.float32)).to(torch.bfloat16)
    return W, X, R


SHAPES = [
    (256, 512, 512),    # one M block, two N blocks: panel 256 wide
    (333, 136, 200),    # ragged M, N (one partial N block) and K (200 = 3 k-blocks + 8)
    (700, 640, 640),    # d = 640 projections: panel 160 wide, 10 k-blocks
    (520, 1920, 640),   # d = 640 MLP fc: panel 192 wide
    (300, 264, 1000),   # K up to 1024: panel 128 wide, 16 k-blocks, ragged N
    (5120, 2048, 512),  # 160 tiles over the pairs: runs cross N blocks
    (512, 16384, 64),   # two tiles per N block: the panel changes at almost every tile
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("bits", [6, 8, 5])
def test_fused_linear_fwd(shape, bits):
    T, N, K = shape
    W, X, R = _case(T, N, K, seed=T + 3 * N + 7 * K + bits)
    Wd, Xd = torch.from_numpy(W).cuda(), X.cuda()
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    qat.qat_linear_fwd(Xd, Y, bits, W=Wd)  # no workspace: the GEMM quantizes W itself
    Y2 = R.cuda()
    qat.qat_linear_fwd(Xd, Y2, bits, W=Wd, residual=Y2)  # residual in place
    q = qat.quantize_weight(Wd, bits)
    Ym = torch.empty_like(Y)
    qat.qat_linear_fwd(Xd, Ym, bits, qw=q)
    torch.cuda.synchronize()
    assert qat.device_error() == 0
    op = o.quantize_weight(W, bits)["operand"]
    ref = o.linear_fwd(op, X.float().numpy())
    assert_close(Y, ref, "Y")
    assert_close(Y2, ref + R.float().numpy(), "Y+residual")
    if N % 256 == 0 and K <= 512:
        assert np.array_equal(bits16(Y), bits16(Ym)), "fused and materialised operand differ"


@pytest.mark.parametrize("d,H,T,act", [(512, 2048, 1000, "relu2"), (512, 1536, 300, "leaky2"),
                                       (640, 1920, 600, "relu2"), (640, 1920, 257, "leaky2")])
def test_fused_mlp_fwd(d, H, T, act):
    """qat_mlp_fwd from the fp32 fc weight and no workspace: the fc GEMM
    quantizes Wfc in its producer and applies the activation in its epilogue;
    proj takes its pre-quantized operand (K = H is longer than a resident
    panel holds)."""
    rng = np.random.default_rng(d + H + T)
    Wfc = (rng.standard_normal((H, d)) * 0.02).astype(np.float32)
    Wproj = (rng.standard_normal((d, H)) * 0.02).astype(np.float32)
    X = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(torch.bfloat16)
    bf = torch.bfloat16
    Y = torch.empty((T, d), dtype=bf, device="cuda")
    pre = torch.empty((T, H), dtype=bf, device="cuda")
    h = torch.empty((T, H), dtype=bf, device="cuda")
    qp = qat.quantize_weight(torch.from_numpy(Wproj).cuda(), 6)
    qat.qat_mlp_fwd(X.cuda(), Y, 6, d, H, Wfc=torch.from_numpy(Wfc).cuda(), qproj=qp,
                    pre_save=pre, h_save=h, act=act)
    torch.cuda.synchronize()
    assert qat.device_error() == 0
    ofc = o.quantize_weight(Wfc, 6)["operand"]
    opj = o.quantize_weight(Wproj, 6)["operand"]
    rpre, rh, rY = o.mlp_fwd(ofc, opj, X.float().numpy(), act=act)
    assert_close(pre, rpre, "pre")
    assert_close(h, rh, "h")
    assert_close(Y, rY, "Y")


def test_fused_degenerate_rows():
    """All-zero rows (amax floored at 1e-12: codes 0) and rows of one repeated
    value next to ordinary rows, through the fused producer."""
    T, N, K = 256, 512, 512
    W, X, _ = _case(T, N, K, seed=11, outliers=False)
    W[3] = 0.0
    W[200] = 0.0125
    W[511] = -3.0
    Wd = torch.from_numpy(W).cuda()
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    qat.qat_linear_fwd(X.cuda(), Y, 6, W=Wd)
    torch.cuda.synchronize()
    ref = o.linear_fwd(o.quantize_weight(W, 6)["operand"], X.float().numpy())
    assert_close(Y, ref, "Y")
    assert np.all(bits16(Y)[:, 3] & 0x7FFF == 0)  # zero weight row -> zero output column
