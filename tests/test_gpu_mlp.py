"""GPU parity of the ReLU^2 MLP (fused relu^2 fc epilogue, fused 2*relu(pre)
backward epilogue) and of its LeakyReLU(0.5)^2 variant, on the int5 / int6 /
int8 grids, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import synthetic as sy
from parity import assert_close

pytestmark = pytest.mark.gpu


def _run(c, d, H, bits=6, raw=False, act="relu2"):
    X, dY = c["X"].cuda(), c["dY"].cuda()
    T = X.shape[0]
    Wfc, Wproj = torch.from_numpy(c["Wfc"]).cuda(), torch.from_numpy(c["Wproj"]).cuda()
    bf = torch.bfloat16
    Y, pre, h = (torch.empty((T, n), dtype=bf, device="cuda") for n in (d, H, H))
    dX = torch.empty((T, d), dtype=bf, device="cuda")
    dWfc = torch.empty((H, d), dtype=torch.float32, device="cuda")
    dWproj = torch.empty((d, H), dtype=torch.float32, device="cuda")
    if raw:
        kw = {"Wfc": Wfc, "Wproj": Wproj}
        wsf = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_FWD, d, H, T, True), dtype=torch.uint8, device="cuda")
        wsb = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_BWD, d, H, T, True), dtype=torch.uint8, device="cuda")
    else:
        kw = {"qfc": qat.quantize_weight(Wfc, bits), "qproj": qat.quantize_weight(Wproj, bits)}
        wsf = None
        wsb = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_BWD, d, H, T, False), dtype=torch.uint8, device="cuda")
    qat.qat_mlp_fwd(X, Y, bits, d, H, pre_save=pre, h_save=h, workspace=wsf, act=act, **kw)
    qat.qat_mlp_bwd(X, pre, h, dY, bits, d, H, dX=dX, dWfc=dWfc, dWproj=dWproj, workspace=wsb,
                    act=act, **kw)
    torch.cuda.synchronize()
    return Y, pre, h, dX, dWfc, dWproj


def _check(c, out, bits=6, act="relu2"):
    qf, qp = o.quantize_weight(c["Wfc"], bits), o.quantize_weight(c["Wproj"], bits)
    X, dY = c["X"].float().numpy(), c["dY"].float().numpy()
    pre, h, Y = o.mlp_fwd(qf["operand"], qp["operand"], X, act)
    dX, dWfc, dWproj = o.mlp_bwd(qf["operand"], qp["operand"], X, pre, h, dY, act)
    for name, g, r in zip(("Y", "pre", "h", "dX", "dWfc", "dWproj"), out, (Y, pre, h, dX, dWfc, dWproj)):
        assert_close(g, r, name)


@pytest.mark.parametrize("raw", [False, True])
def test_mlp_small_ragged(raw):
    c = sy.mlp_case(T=1000)
    _check(c, _run(c, 512, 1536, raw=raw))


def test_mlp_odd_dims():
    c = sy.mlp_case(d=136, H=264, T=333, seed=4)
    _check(c, _run(c, 136, 264))


def test_mlp_cfg2_full_size():
    """The 11-layer record's MLP block at 8x1024 tokens, every element."""
    c = sy.mlp_case(T=8192)
    _check(c, _run(c, 512, 1536))
    assert qat.device_error() == 0


@pytest.mark.parametrize("bits", [5, 8])
@pytest.mark.parametrize("act", ["relu2", "leaky2"])
def test_mlp_bits_and_activation(bits, act):
    """int5 / int8 grids and LeakyReLU(0.5)^2, raw fp32 weights and cached
    operands, ragged token count spanning several tiles."""
    c = sy.mlp_case(T=1000, seed=7)
    _check(c, _run(c, 512, 1536, bits=bits, act=act), bits=bits, act=act)
    _check(c, _run(c, 512, 1536, bits=bits, raw=True, act=act), bits=bits, act=act)


def test_mlp_leaky2_full_size():
    """LeakyReLU(0.5)^2 MLP at 8x1024 tokens (int5, the all-int5 configuration),
    every element."""
    c = sy.mlp_case(T=8192, seed=8)
    _check(c, _run(c, 512, 1536, bits=5, act="leaky2"), bits=5, act="leaky2")
    assert qat.device_error() == 0


@pytest.mark.parametrize("alias", [False, True])
def test_mlp_bwd_dx_residual(alias):
    """dX = dpre . Wfc_q + residual (the gradient around a residual MLP), the
    residual added before the bf16 rounding, also in place in dX."""
    d, H, T = 640, 1920, 700
    c = sy.mlp_case(d=d, H=H, T=T, seed=9)
    Rs = sy.act_bf16(np.random.default_rng(9), T, d, std=0.01)
    qf = qat.quantize_weight(torch.from_numpy(c["Wfc"]).cuda(), 6)
    qp = qat.quantize_weight(torch.from_numpy(c["Wproj"]).cuda(), 6)
    bf = torch.bfloat16
    X, dY = c["X"].cuda(), c["dY"].cuda()
    Y, pre, h = (torch.empty((T, n), dtype=bf, device="cuda") for n in (d, H, H))
    Rd = Rs.cuda()
    dX = Rd if alias else torch.empty((T, d), dtype=bf, device="cuda")
    ws = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_BWD, d, H, T, False), dtype=torch.uint8,
                     device="cuda")
    qat.qat_mlp_fwd(X, Y, 6, d, H, qfc=qf, qproj=qp, pre_save=pre, h_save=h)
    qat.qat_mlp_bwd(X, pre, h, dY, 6, d, H, qfc=qf, qproj=qp, dX=dX, dX_residual=Rd, workspace=ws)
    torch.cuda.synchronize()
    rf, rp = o.quantize_weight(c["Wfc"], 6), o.quantize_weight(c["Wproj"], 6)
    Xn = c["X"].float().numpy()
    p_, h_, _ = o.mlp_fwd(rf["operand"], rp["operand"], Xn)
    rdX = o.mlp_bwd(rf["operand"], rp["operand"], Xn, p_, h_, c["dY"].float().numpy())[0]
    assert_close(dX, rdX + Rs.float().numpy(), "dX + residual")
    assert qat.device_error() == 0


def test_mlp_bwd_dpre_save():
    """dpre written to the caller's buffer (no workspace): dh * act'(pre) at the
    single-op tolerance, and dX / dWfc / dWproj as with the workspace."""
    d, H, T = 512, 2048, 1000
    c = sy.mlp_case(d=d, H=H, T=T, seed=10)
    qf = qat.quantize_weight(torch.from_numpy(c["Wfc"]).cuda(), 6)
    qp = qat.quantize_weight(torch.from_numpy(c["Wproj"]).cuda(), 6)
    bf = torch.bfloat16
    X, dY = c["X"].cuda(), c["dY"].cuda()
    Y, pre, h, dpre = (torch.empty((T, n), dtype=bf, device="cuda") for n in (d, H, H, H))
    dX = torch.empty((T, d), dtype=bf, device="cuda")
    dWfc = torch.empty((H, d), dtype=torch.float32, device="cuda")
    dWproj = torch.empty((d, H), dtype=torch.float32, device="cuda")
    qat.qat_mlp_fwd(X, Y, 6, d, H, qfc=qf, qproj=qp, pre_save=pre, h_save=h)
    qat.qat_mlp_bwd(X, pre, h, dY, 6, d, H, qfc=qf, qproj=qp, dX=dX, dWfc=dWfc, dWproj=dWproj,
                    dpre_save=dpre)
    torch.cuda.synchronize()
    rf, rp = o.quantize_weight(c["Wfc"], 6), o.quantize_weight(c["Wproj"], 6)
    Xn, dYn = c["X"].float().numpy(), c["dY"].float().numpy()
    p_, h_, _ = o.mlp_fwd(rf["operand"], rp["operand"], Xn)
    rdpre = (dYn.astype(np.float64) @ rp["operand"]) * o.act_grad(p_)
    assert_close(dpre, rdpre, "dpre")
    rdX, rdWfc, rdWproj = o.mlp_bwd(rf["operand"], rp["operand"], Xn, p_, h_, dYn)
    assert_close(dX, rdX, "dX")
    assert_close(dWfc, rdWfc, "dWfc")
    assert_close(dWproj, rdWproj, "dWproj")
    assert qat.device_error() == 0
