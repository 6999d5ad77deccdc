"""GPU parity of Noisy QAT ("Depth Recurrence + Mixed-Precision Quant",
"幸存发现 1"): the noisy bf16 operand bit-exact against the oracle's Philox and
fp32 arithmetic, the linear forward / backward through it, and the recurrent
core with fresh noise per application."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat, steps
from quantization_aware_tiny_b200 import synthetic as sy
from parity import (assert_close, assert_close_chain, bits16, chain_allowance, core_sums,
                    rounding_noise_allowance)

pytestmark = pytest.mark.gpu

SEEDS = [(0, 0), (1234, 7), ((0xDEADBEEF << 32) | 0x1234567, (0xFFFFFFFF << 32) | 3)]


@pytest.mark.parametrize("seed,offset", SEEDS)
@pytest.mark.parametrize("bits", [8, 5])
def test_noisy_operand_bit_exact(seed, offset, bits):
    """Noise at the int8 step (bits 8) and at the int5 step (bits 5)."""
    rng = np.random.default_rng(31)
    for shape in ((512, 512), (200, 136), (64, 4104), (1280, 640)):
        W = (rng.standard_normal(shape) * 0.02).astype(np.float32)
        q = qat.noisy_weight(torch.from_numpy(W).cuda(), seed, offset, bits=bits)
        torch.cuda.synchronize()
        ref = o.noisy_weight(W, seed, offset, bits)
        assert np.array_equal(bits16(q.operand), ref["operand_bits"]), shape
        assert np.array_equal(q.scales.cpu().numpy(), ref["scales"]), shape
    assert qat.device_error() == 0


def test_noisy_linear_fwd_bwd():
    c = sy.linear_case(N=512, K=512, T=300, seed=2, with_dy=True)
    W = torch.from_numpy(c["W"]).cuda()
    q = qat.noisy_weight(W, 99, 5)
    T = 300
    Y = torch.empty((T, 512), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((T, 512), dtype=torch.bfloat16, device="cuda")
    dW = torch.empty((512, 512), dtype=torch.float32, device="cuda")
    qat.qat_linear_fwd(c["X"].cuda(), Y, 8, qw=q)
    qat.qat_linear_bwd(c["X"].cuda(), c["dY"].cuda(), 8, qw=q, dX=dX, dW=dW)
    torch.cuda.synchronize()
    op = o.noisy_weight(c["W"], 99, 5)["operand"]
    X, dY = c["X"].float().numpy(), c["dY"].float().numpy()
    assert_close(Y, o.linear_fwd(op, X), "Y")
    rdX, rdW = o.linear_bwd(op, X, dY)
    assert_close(dX, rdX, "dX")
    assert_close(dW, rdW, "dW")


def _noisy_core(c, bits=6, act="relu2"):
    dev = {k: torch.from_numpy(c[k]).cuda() for k in ("Wq", "Wk", "Wv", "Wo", "Wfc", "Wproj")}
    core = steps.RecurrentCore(dev["Wq"], dev["Wk"], dev["Wv"], dev["Wo"], dev["Wfc"], dev["Wproj"],
                               bits=bits, act=act)
    Ws = [np.concatenate([c["Wq"], c["Wk"], c["Wv"]]), c["Wo"], c["Wfc"], c["Wproj"]]
    return core, Ws


def test_noisy_recurrent_core():
    c = sy.recurrent_core_case(T=300)
    core, Ws = _noisy_core(c)
    x = c["X"].cuda()
    core.forward(x, 3, noise=(2024, 100))
    torch.cuda.synchronize()
    ref, saved = o.core_fwd_apps(o.noisy_core_ops(Ws, 3, 2024, 100), c["X"].float().numpy(), 640)
    assert_close_chain(x, ref, chain_allowance(core_sums(saved)), "noisy core, 3 applications")
    assert qat.device_error() == 0


def test_noisy_recurrent_core_per_application():
    """Each Noisy-QAT application from the oracle's state before it, at the
    single-op tolerance: application r draws at offsets offset + 4*r + k."""
    c = sy.recurrent_core_case(T=300, seed=6)
    core, Ws = _noisy_core(c)
    apps = o.noisy_core_ops(Ws, 3, 31, 8)
    _, saved = o.core_fwd_apps(apps, c["X"].float().numpy(), 640)
    for r, s in enumerate(saved):
        x = torch.from_numpy(s["x"].astype(np.float32)).to(torch.bfloat16).cuda()
        out = core.forward_train(x, 1, noise=(31, 8 + 4 * r))
        torch.cuda.synchronize()
        assert_close(out, s["out"], "noisy application %d" % r)
    assert qat.device_error() == 0


def test_noisy_recurrent_core_int5_leaky2():
    """An all-int5 core (noise at the int5 step, as the write-up proposes for an
    int5 export) with the LeakyReLU(0.5)^2 MLP."""
    c = sy.recurrent_core_case(T=300, seed=3)
    core, Ws = _noisy_core(c, bits=5, act="leaky2")
    x = c["X"].cuda()
    core.forward(x, 2, noise=(77, 4))
    torch.cuda.synchronize()
    ref, saved = o.core_fwd_apps(o.noisy_core_ops(Ws, 2, 77, 4, bits=5), c["X"].float().numpy(),
                                 640, act="leaky2")
    assert_close_chain(x, ref, chain_allowance(core_sums(saved)),
                       "noisy int5 leaky core, 2 applications")
    assert qat.device_error() == 0


def test_noisy_recurrent_core_bwd():
    """Noisy-QAT core forward and backward through R = 3 applications: the
    backward of application r uses that application's noisy operands (the
    noise carries no gradient)."""
    T = 300
    c = sy.recurrent_core_case(T=T, seed=4)
    core, Ws = _noisy_core(c)
    dY = sy.act_bf16(np.random.default_rng(14), T, 640, std=sy.DY_STD)
    out = core.forward_train(c["X"].cuda(), 3, noise=(5, 40))
    dX = core.backward(dY.cuda())
    torch.cuda.synchronize()
    ref = o.recurrent_core_bwd_noisy(Ws, c["X"].float().numpy(), dY.float().numpy(), 3, 640, 5, 40)
    ops = o.noisy_core_ops(Ws, 3, 5, 40)
    _, sx = o.core_fwd_apps(ops, c["X"].float().numpy(), 640, exact=True)
    ex = o.core_bwd_apps(ops, sx, dY.float().numpy(), 640, exact=True)[1]
    assert_close_chain(out, ref["out"], chain_allowance(core_sums(ref["saved"])), "noisy core: out")
    assert_close(dX, ref["dX"], "noisy core: dX")
    for k in ("qkv", "o", "fc", "proj"):
        assert_close_chain(getattr(core, "dW" + k), ref["dW" + k],
                           rounding_noise_allowance(ref["dW" + k], ex[k]), "noisy core: dW" + k)
    assert qat.device_error() == 0
