"""GPU parity of the multi-call paths against the oracle: the depth-recurrent
core (quantize once, apply R=3 times) and the tied-head + MLP training step,
at small sizes element by element and at the benchmark's full sizes on
sampled outputs the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import steps
from quantization_aware_tiny_b200 import synthetic as sy
from parity import (assert_close, assert_close_chain, chain_allowance, core_sums,
                    rounding_noise_allowance, to_np)

pytestmark = pytest.mark.gpu


def _core(c, bits=6, act="relu2"):
    dev = {k: torch.from_numpy(c[k]).cuda() for k in ("Wq", "Wk", "Wv", "Wo", "Wfc", "Wproj")}
    return steps.RecurrentCore(dev["Wq"], dev["Wk"], dev["Wv"], dev["Wo"], dev["Wfc"], dev["Wproj"], bits,
                               act=act)


def _core_oracle(c, bits=6):
    q = {"qkv": o.quantize_weight(np.concatenate([c["Wq"], c["Wk"], c["Wv"]]), bits),
         "o": o.quantize_weight(c["Wo"], bits), "fc": o.quantize_weight(c["Wfc"], bits),
         "proj": o.quantize_weight(c["Wproj"], bits)}
    return q


def _core_ops(q):
    return (q["qkv"], q["o"], q["fc"], q["proj"])


def test_recurrent_core_small():
    c = sy.recurrent_core_case(T=300)
    core = _core(c)
    x = c["X"].cuda()
    n0 = qat.launch_count()
    core.forward(x, 3)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 3 * 4  # no re-quantization inside the loop
    q = _core_oracle(c)
    ref, saved = o.core_fwd_apps([_core_ops(q)] * 3, c["X"].float().numpy(), 640)
    assert_close_chain(x, ref, chain_allowance(core_sums(saved)), "x after 3 applications")


@pytest.mark.parametrize("bits,act", [(6, "relu2"), (5, "leaky2")])
def test_recurrent_core_per_application(bits, act):
    """Each application on its own, from the oracle's bf16 state before it:
    the output state and the kept activations (qkv, x1, pre, h) at the
    single-op tolerance, with no allowance for a chain."""
    c = sy.recurrent_core_case(T=300, seed=2)
    core = _core(c, bits, act)
    q = _core_oracle(c, bits)
    _, saved = o.core_fwd_apps([_core_ops(q)] * 3, c["X"].float().numpy(), 640, act)
    for r, s in enumerate(saved):
        x = torch.from_numpy(s["x"].astype(np.float32)).to(torch.bfloat16).cuda()
        out = core.forward_train(x, 1)
        torch.cuda.synchronize()
        assert_close(out, s["out"], "application %d: out" % r)
        for k in ("qkv", "x1", "pre", "h"):
            assert_close(core._saved(0)[k], s[k], "application %d: %s" % (r, k))
        x1 = x.clone()
        core.forward(x1, 1)  # the inference forward, in place
        assert_close(x1, s["out"], "application %d: in-place forward" % r)
    assert qat.device_error() == 0


@pytest.mark.parametrize("bits,act", [(5, "relu2"), (5, "leaky2"), (6, "leaky2")])
def test_recurrent_core_int5_and_leaky2(bits, act):
    """The all-int5 core (MLP_INT5 + ATTN_INT5) and the LeakyReLU(0.5)^2 MLP."""
    c = sy.recurrent_core_case(T=300, seed=5)
    core = _core(c, bits, act)
    x = c["X"].cuda()
    core.forward(x, 3)
    torch.cuda.synchronize()
    q = _core_oracle(c, bits)
    ref, saved = o.core_fwd_apps([_core_ops(q)] * 3, c["X"].float().numpy(), 640, act)
    assert_close_chain(x, ref, chain_allowance(core_sums(saved)), "x after 3 applications")


def test_recurrent_cache_matches_fresh_quantization():
    c = sy.recurrent_core_case(T=8)
    core = _core(c)
    q = _core_oracle(c)
    torch.cuda.synchronize()
    for name, g in (("qkv", core.q_qkv), ("o", core.q_o), ("fc", core.q_fc), ("proj", core.q_proj)):
        assert np.array_equal(g.operand.cpu().view(torch.int16).numpy().view(np.uint16),
                              o.bf16_bits(q[name]["operand"].astype(np.float32))), name


def test_recurrent_core_full_size_sampled_rows():
    """3x3 core at d=640, 16x1024 tokens, R=3: rows evolve independently (no
    attention), so the oracle runs the sampled rows through all three
    applications."""
    c = sy.recurrent_core_case(T=16384)
    core = _core(c)
    x = c["X"].cuda()
    core.forward(x, 3)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(16384, 64, replace=False)
    rows = np.concatenate([rows, [0, 16383]])
    q = _core_oracle(c)
    ref, saved = o.core_fwd_apps([_core_ops(q)] * 3, c["X"].float().numpy()[rows], 640)
    assert_close_chain(to_np(x)[rows], ref, chain_allowance(core_sums(saved)), "sampled rows")
    assert qat.device_error() == 0


# ------------------------------------------------- recurrent core backward

def _grads(core):
    return {k: getattr(core, k).clone() for k in ("dWqkv", "dWo", "dWfc", "dWproj")}


def _core_bwd_check(grads, ref, exact, x_out, dX, what, rows=None):
    """The chained forward + backward: the output state within the chain
    allowance, dX at the single-op tolerance, the summed weight gradients
    within the chain's bf16 rounding noise (measured by the oracle as its
    rounded run against its exact run); relative Frobenius <= 5e-3 for all."""
    sel = (lambda a: a) if rows is None else (lambda a: np.asarray(a)[rows])
    assert_close_chain(sel(to_np(x_out)), sel(ref["out"]),
                       chain_allowance([sel(u) for u in core_sums(ref["saved"])]), what + ": out")
    assert_close(sel(to_np(dX)), sel(ref["dX"]), what + ": dX")
    for k in ("dWqkv", "dWo", "dWfc", "dWproj"):
        assert_close_chain(grads[k], ref[k], rounding_noise_allowance(ref[k], exact[k]),
                           what + ": " + k)
    d = grads["dWo"].shape[0]
    assert torch.count_nonzero(grads["dWqkv"][d:]).item() == 0  # k, v: no gradient


@pytest.mark.parametrize("bits,act", [(6, "relu2"), (5, "leaky2")])
def test_recurrent_core_bwd_small(bits, act):
    """Forward (activations kept) and backward through R = 3 applications in
    reverse, the shared weights' gradients summed over the three uses."""
    T = 300
    c = sy.recurrent_core_case(T=T, seed=1)
    dY = sy.act_bf16(np.random.default_rng(11), T, 640, std=sy.DY_STD)
    core = _core(c, bits, act)
    x = c["X"].cuda()
    n0 = qat.launch_count()
    out = core.forward_train(x, 3)
    dX = core.backward(dY.cuda())
    torch.cuda.synchronize()
    # 4 GEMMs per application forward; 4 per application for the gradient's
    # chain backward (dpre, dx1, dq, dx), then one GEMM per shared weight over
    # all 3 x 300 token uses
    assert qat.launch_count() - n0 == 3 * 4 + 3 * 4 + 4
    assert torch.equal(x, c["X"].cuda())  # the input state is left as it is
    q = _core_oracle(c, bits)
    args = (*_core_ops(q), c["X"].float().numpy(), dY.float().numpy(), 3, 640, act)
    ref = o.recurrent_core_bwd(*args)
    exact = o.recurrent_core_bwd(*args, exact=True)
    _core_bwd_check(_grads(core), ref, exact, out, dX, "R=3")
    assert qat.device_error() == 0


@pytest.mark.parametrize("T,R,d,H,bits,act", [(257, 1, 640, 1920, 6, "relu2"),
                                               (1000, 2, 512, 1536, 8, "relu2"),
                                               (513, 3, 512, 2048, 5, "leaky2")])
def test_recurrent_core_bwd_shapes(T, R, d, H, bits, act):
    """Forward + backward at other shapes: ragged token counts (not multiples
    of the 256-row tiles), R = 1 and 2, the d = 512 core (8 query / 4 KV heads
    of dim 64) with 3x and 4x MLPs, the int8 and int5 grids, LeakyReLU(0.5)^2."""
    c = sy.recurrent_core_case(d=d, H=H, T=T, seed=T)
    dY = sy.act_bf16(np.random.default_rng(T), T, d, std=sy.DY_STD)
    core = _core(c, bits, act)
    out = core.forward_train(c["X"].cuda(), R)
    dX = core.backward(dY.cuda())
    torch.cuda.synchronize()
    q = _core_oracle(c, bits)
    args = (*_core_ops(q), c["X"].float().numpy(), dY.float().numpy(), R, d, act)
    ref = o.recurrent_core_bwd(*args)
    exact = o.recurrent_core_bwd(*args, exact=True)
    _core_bwd_check(_grads(core), ref, exact, out, dX, "T=%d R=%d d=%d" % (T, R, d))
    assert qat.device_error() == 0


def test_recurrent_core_bwd_accumulates_across_calls():
    """backward(accumulate=True) adds this call's summed gradients to the
    held ones (gradient accumulation over micro-batches): two micro-batches
    give the sum of their oracle gradients."""
    T = 300
    cs = [sy.recurrent_core_case(T=T, seed=s) for s in (21, 22)]
    core = _core(cs[0])
    dYs = [sy.act_bf16(np.random.default_rng(30 + i), T, 640, std=sy.DY_STD) for i in range(2)]
    for i, c in enumerate(cs):
        core.forward_train(c["X"].cuda(), 2)
        core.backward(dYs[i].cuda(), accumulate=i > 0)
    torch.cuda.synchronize()
    q = _core_oracle(cs[0])
    refs = [o.recurrent_core_bwd(*_core_ops(q), c["X"].float().numpy(), dY.float().numpy(), 2, 640)
            for c, dY in zip(cs, dYs)]
    exs = [o.recurrent_core_bwd(*_core_ops(q), c["X"].float().numpy(), dY.float().numpy(), 2, 640,
                                exact=True) for c, dY in zip(cs, dYs)]
    for k in ("dWqkv", "dWo", "dWfc", "dWproj"):
        ref = refs[0][k] + refs[1][k]
        noise = np.hypot(rounding_noise_allowance(refs[0][k], exs[0][k]),
                         rounding_noise_allowance(refs[1][k], exs[1][k]))
        assert_close_chain(getattr(core, k), ref, noise, "accumulated " + k)
    assert qat.device_error() == 0


def test_recurrent_core_bwd_zero_tokens():
    """No tokens: the forward returns an empty state, dX is empty and every
    weight gradient is zero (no token uses to sum)."""
    c = sy.recurrent_core_case(T=8)
    core = _core(c)
    x = torch.empty((0, 640), dtype=torch.bfloat16, device="cuda")
    out = core.forward_train(x, 3)
    dX = core.backward(torch.empty((0, 640), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert out.shape == (0, 640) and dX.shape == (0, 640)
    for k in ("dWqkv", "dWo", "dWfc", "dWproj"):
        assert torch.count_nonzero(getattr(core, k)).item() == 0, k
    assert qat.device_error() == 0


def test_recurrent_core_bwd_per_application():
    """Each application's backward on its own, from the oracle's saved bf16
    activations and incoming gradient: dx and the application's weight
    gradients at the single-op tolerance."""
    T = 300
    c = sy.recurrent_core_case(T=T, seed=3)
    dY = sy.act_bf16(np.random.default_rng(12), T, 640, std=sy.DY_STD)
    core = _core(c)
    q = _core_oracle(c)
    ops = _core_ops(q)
    ref = o.recurrent_core_bwd(*ops, c["X"].float().numpy(), dY.float().numpy(), 3, 640)
    bf = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).cuda()
    dx = torch.empty((T, 640), dtype=torch.bfloat16, device="cuda")
    for r, s in enumerate(ref["saved"]):
        sd = {k: bf(s[k]) for k in ("x", "qkv", "x1", "pre", "h")}
        sd["ops"] = (core.q_qkv, core.q_o, core.q_fc, core.q_proj)
        core.backward_application(sd, bf(ref["grads"][r]), dx, accumulate=False)
        torch.cuda.synchronize()
        gx, dW, _ = o.core_application_bwd(ops, s, ref["grads"][r], 640)
        assert_close(dx, gx, "application %d: dx" % r)
        for k, name in (("qkv", "dWqkv"), ("o", "dWo"), ("fc", "dWfc"), ("proj", "dWproj")):
            assert_close(getattr(core, name), dW[k], "application %d: %s" % (r, name))
    # accumulate over the three applications into the same gradients
    for r, s in enumerate(ref["saved"]):
        sd = {k: bf(s[k]) for k in ("x", "qkv", "x1", "pre", "h")}
        sd["ops"] = (core.q_qkv, core.q_o, core.q_fc, core.q_proj)
        core.backward_application(sd, bf(ref["grads"][r]), dx, accumulate=r > 0)
    torch.cuda.synchronize()
    for k in ("dWqkv", "dWo", "dWfc", "dWproj"):
        assert_close(getattr(core, k), ref[k], "summed over applications: " + k)
    assert qat.device_error() == 0


@pytest.fixture(scope="module")
def full_core():
    """The 3x3 core at d=640, 16x1024 tokens, R=3, forward (activations kept)
    and backward as the benchmark launches them, and the oracle's rounded
    run of the same."""
    T = 16384
    c = sy.recurrent_core_case(T=T)
    dY = sy.act_bf16(np.random.default_rng(13), T, 640, std=sy.DY_STD)
    core = _core(c)
    out = core.forward_train(c["X"].cuda(), 3).clone()
    dX = core.backward(dY.cuda()).clone()
    grads = _grads(core)
    torch.cuda.synchronize()
    q = _core_oracle(c)
    args = (*_core_ops(q), c["X"].float().numpy(), dY.float().numpy(), 3, 640)
    ref = o.recurrent_core_bwd(*args)
    return c, core, q, args, ref, out, dX, grads


def test_recurrent_core_bwd_full_size_chained(full_core):
    """Chained at full size: the output state and dX on sampled rows (rows
    are independent without attention), every entry of the four summed
    weight gradients within the chain's rounding noise."""
    c, core, q, args, ref, out, dX, grads = full_core
    exact = o.recurrent_core_bwd(*args, exact=True)
    rows = np.concatenate([np.random.default_rng(4).choice(16384, 64, replace=False), [0, 16383]])
    _core_bwd_check(grads, ref, exact, out, dX, "R=3 full size", rows=rows)
    assert qat.device_error() == 0


def test_recurrent_core_per_application_full_size(full_core):
    """Each application at full size on its own, from the oracle's bf16
    inputs, at the single-op tolerance: the forward's output state on sampled
    rows, the backward's dx on sampled rows and every entry of that
    application's four weight gradients."""
    c, core, q, args, ref, out, dX, grads = full_core
    ops = _core_ops(q)
    T = 16384
    rows = np.concatenate([np.random.default_rng(5).choice(T, 64, replace=False), [0, T - 1]])
    bf = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).cuda()
    dx = torch.empty((T, 640), dtype=torch.bfloat16, device="cuda")
    for r, s in enumerate(ref["saved"]):
        x = bf(s["x"])
        y = core.forward_train(x, 1)
        torch.cuda.synchronize()
        assert_close(to_np(y)[rows], s["out"][rows], "application %d: out" % r)
        sd = {k: bf(s[k]) for k in ("x", "qkv", "x1", "pre", "h")}
        sd["ops"] = (core.q_qkv, core.q_o, core.q_fc, core.q_proj)
        core.backward_application(sd, bf(ref["grads"][r]), dx, accumulate=False)
        torch.cuda.synchronize()
        gx, dW, _ = o.core_application_bwd(ops, s, ref["grads"][r], 640)
        assert_close(to_np(dx)[rows], gx[rows], "application %d: dx" % r)
        for k, name in (("qkv", "dWqkv"), ("o", "dWo"), ("fc", "dWfc"), ("proj", "dWproj")):
            assert_close(getattr(core, name), dW[k], "application %d: %s" % (r, name))
        del sd
    assert qat.device_error() == 0


def _head_step(c):
    dev = lambda k: torch.from_numpy(c[k]).cuda()
    s = steps.HeadMlpStep(dev("Wemb"), dev("Wfc"), dev("Wproj"), c["X"].shape[0])
    X, dL = c["X"].cuda(), c["dLogits"].cuda()
    s.step(X, dL)
    torch.cuda.synchronize()
    return s


def _head_q(c):
    return o.quantize_weight(c["Wemb"], 8), o.quantize_weight(c["Wfc"], 6), o.quantize_weight(c["Wproj"], 6)


def test_head_mlp_step_small():
    c = sy.head_mlp_case(T=300)
    s = _head_step(c)
    qe, qf, qp = _head_q(c)
    ref = o.head_mlp_step(qe, qf, qp, c["X"].float().numpy(), c["dLogits"].float().numpy())
    for name, g in (("Z", s.Z), ("logits", s.logits), ("dZ", s.dZ), ("dX", s.dX),
                    ("dWemb", s.dWemb), ("dWfc", s.dWfc), ("dWproj", s.dWproj)):
        assert_close(g, ref[name], name)


def test_head_mlp_step_4096_tokens_every_output():
    """The throughput configuration at its smallest token count (4,096): every
    output and every gradient entry against the oracle."""
    c = sy.head_mlp_case(T=4096, seed=3)
    s = _head_step(c)
    qe, qf, qp = _head_q(c)
    ref = o.head_mlp_step(qe, qf, qp, c["X"].float().numpy(), c["dLogits"].float().numpy())
    for name, g in (("Z", s.Z), ("logits", s.logits), ("dZ", s.dZ), ("dX", s.dX),
                    ("dWemb", s.dWemb), ("dWfc", s.dWfc), ("dWproj", s.dWproj)):
        assert_close(g, ref[name], name)
    assert qat.device_error() == 0


def test_head_mlp_step_16384_tokens_sampled():
    """16,384 tokens: per-token outputs on sampled rows; weight-gradient entries
    on sampled rows and columns, each summed over all tokens by the oracle."""
    T = 16384
    c = sy.head_mlp_case(T=T, seed=4)
    s = _head_step(c)
    qe, qf, qp = _head_q(c)
    rows = np.concatenate([np.random.default_rng(2).choice(T, 40, replace=False), [0, T - 1]])
    Xall, dLall = c["X"].float().numpy(), c["dLogits"].float().numpy()
    ref = o.head_mlp_step(qe, qf, qp, Xall[rows], dLall[rows])
    for name, g in (("Z", s.Z), ("logits", s.logits), ("dZ", s.dZ), ("dX", s.dX)):
        assert_close(to_np(g)[rows], ref[name], name)
    # dWemb[v, k] = sum_t dL[t, v] Z[t, k], with Z the MLP output of every token
    Z = o.linear_fwd(qp["operand"], o.relu2(o.linear_fwd(qf["operand"], Xall)))
    vs, ks = [0, 4095, 8191], [0, 255, 511]
    assert_close(to_np(s.dWemb)[np.ix_(vs, ks)], dLall[:, vs].T @ Z[:, ks], "dWemb sampled")
    assert qat.device_error() == 0


@pytest.fixture(scope="module")
def full_head():
    c = sy.head_mlp_case(T=65536)
    s = _head_step(c)
    return c, s


def test_head_mlp_step_full_size_rows(full_head):
    """T=65,536 step as the benchmark launches it: per-token outputs on sampled rows."""
    c, s = full_head
    qe, qf, qp = _head_q(c)
    rows = np.concatenate([np.random.default_rng(1).choice(65536, 48, replace=False), [0, 65535]])
    X = c["X"].float().numpy()[rows]
    dL = c["dLogits"].float().numpy()[rows]
    ref = o.head_mlp_step(qe, qf, qp, X, dL)
    for name, g in (("Z", s.Z), ("logits", s.logits), ("dZ", s.dZ), ("dX", s.dX)):
        assert_close(to_np(g)[rows], ref[name], name)
    # dWproj[n, j] = sum_t dZ[t, n] h[t, j]: columns computed over all tokens
    Xall, dLall = c["X"].float().numpy(), c["dLogits"].float().numpy()
    ns, js = [0, 17, 511], [0, 1000, 2047]
    dZ_cols = o.linear_fwd(qe["operand"][:, ns].T, dLall)          # dZ[:, ns] = dL . Wemb_q[:, ns]
    h_cols = o.relu2(o.linear_fwd(qf["operand"][js], Xall))         # h[:, js]
    assert_close(to_np(s.dWproj)[np.ix_(ns, js)], dZ_cols.T @ h_cols, "dWproj sampled")
    assert qat.device_error() == 0


def test_head_bwd_full_size_sampled():
    """Head backward at T=65,536 (the benchmark's launch configuration) on
    generator inputs: sampled dWemb entries and dX rows."""
    c = sy.head_mlp_case(T=65536)
    Z = sy.act_bf16(np.random.default_rng(77), 65536, 512, std=0.25)
    q = qat.quantize_weight(torch.from_numpy(c["Wemb"]).cuda(), 8)
    dX = torch.empty((65536, 512), dtype=torch.bfloat16, device="cuda")
    dW = torch.empty((8192, 512), dtype=torch.float32, device="cuda")
    qat.qat_linear_bwd(Z.cuda(), c["dLogits"].cuda(), 8, qw=q, dX=dX, dW=dW)
    torch.cuda.synchronize()
    op = o.quantize_weight(c["Wemb"], 8)["operand"]
    dL, Zn = c["dLogits"].float().numpy(), Z.float().numpy()
    ns, ks = [0, 5, 4095, 8191], [0, 129, 511]
    assert_close(to_np(dW)[np.ix_(ns, ks)], dL[:, ns].astype(np.float64).T @ Zn[:, ks], "dWemb sampled")
    rows = [0, 12345, 65535]
    assert_close(to_np(dX)[rows], o.linear_bwd(op, Zn[rows], dL[rows])[0], "dX rows")


def test_mlp_bwd_full_size_sampled():
    """MLP backward at T=65,536 on generator inputs: sampled dWfc / dWproj entries."""
    c = sy.head_mlp_case(T=65536)
    dY = sy.act_bf16(np.random.default_rng(78), 65536, 512, std=0.02)
    X = c["X"].cuda()
    qf = qat.quantize_weight(torch.from_numpy(c["Wfc"]).cuda(), 6)
    qp = qat.quantize_weight(torch.from_numpy(c["Wproj"]).cuda(), 6)
    bf = torch.bfloat16
    T, d, H = 65536, 512, 2048
    Y, pre, h = (torch.empty((T, n), dtype=bf, device="cuda") for n in (d, H, H))
    dX = torch.empty((T, d), dtype=bf, device="cuda")
    dWfc = torch.empty((H, d), dtype=torch.float32, device="cuda")
    dWproj = torch.empty((d, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_BWD, d, H, T, False), dtype=torch.uint8, device="cuda")
    qat.qat_mlp_fwd(X, Y, 6, d, H, qfc=qf, qproj=qp, pre_save=pre, h_save=h)
    qat.qat_mlp_bwd(X, pre, h, dY.cuda(), 6, d, H, qfc=qf, qproj=qp, dX=dX, dWfc=dWfc,
                    dWproj=dWproj, workspace=ws)
    torch.cuda.synchronize()
    rf, rp = o.quantize_weight(c["Wfc"], 6), o.quantize_weight(c["Wproj"], 6)
    Xn, dYn = c["X"].float().numpy(), dY.float().numpy()
    ns, ks = [0, 777, 2047], [0, 300, 511]
    pre_c = o.linear_fwd(rf["operand"][ns], Xn)                       # pre[:, ns]
    dh_c = o.linear_fwd(rp["operand"][:, ns].T, dYn)                  # dh[:, ns] = dY . Wproj_q[:, ns]
    dpre_c = dh_c * 2.0 * np.maximum(pre_c, 0.0)
    assert_close(to_np(dWfc)[np.ix_(ns, ks)], dpre_c.T @ Xn[:, ks], "dWfc sampled")
    h_c = o.relu2(o.linear_fwd(rf["operand"][[5, 1999]], Xn))
    assert_close(to_np(dWproj)[np.ix_(ks, [5, 1999])], dYn[:, ks].astype(np.float64).T @ h_c, "dWproj sampled")
    rows = [3, 40000]
    r = o.mlp_bwd(rf["operand"], rp["operand"], Xn[rows], *o.mlp_fwd(rf["operand"], rp["operand"], Xn[rows])[:2], dYn[rows])
    assert_close(to_np(dX)[rows], r[0], "dX rows")
    assert qat.device_error() == 0
