"""The library's calls inside CUDA graphs.  Every entry point launches only on
the stream it is given and allocates nothing, so a captured sequence (the
grouped export of a state dict; a whole QAT training step with its memsets,
programmatic-dependent GEMM launches and split-K reductions) replays to the
results of the direct calls: bit for bit where the kernels are deterministic
(codes, scales, passthrough values, forward GEMM outputs), within the GEMM
tolerance against the oracle where fp32 reductions add partial sums in an
unspecified order (weight gradients).  A replay reads its input buffers as
they are at replay time."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import export as qexport
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import steps
from quantization_aware_tiny_b200 import synthetic as sy
from parity import assert_close, bits16

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Run fn(stream) once directly, then capture it into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def test_export_state_dict_graph_replay_bit_exact():
    sd = sy.state_dict_case(n_layers=2, seed=4)
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in sd.items()}
    held = {}

    def run(st):
        held["out"] = qexport.export_state_dict(dev, stream=st)

    g = _capture(run)
    out = held["out"]  # the outputs the captured launch writes
    for v in out.values():  # overwrite them, so only the replay can restore them
        for key in ("codes", "values", "scale16"):
            if key in v:
                v[key].view(torch.uint8).fill_(0xA5)
    n0 = qat.launch_count()
    g.replay()
    torch.cuda.synchronize()
    assert qat.launch_count() == n0  # the replay goes through the graph, not the library
    assert qat.device_error() == 0
    ref = o.export_state_dict(sd)
    for k, r in ref.items():
        v = out[k]
        assert v["kind"] == r["kind"], k
        if r["kind"] == "fp16":
            assert np.array_equal(bits16(v["values"]).reshape(-1), r["bits16"].reshape(-1)), k
        else:
            assert np.array_equal(v["codes"].cpu().numpy(), r["codes"]), k
            assert np.array_equal(bits16(v["scale16"]), r["scale16"]), k


def test_head_mlp_step_graph_replay():
    T = 1000
    c = sy.head_mlp_case(T=T, seed=9)
    dev = lambda k: torch.from_numpy(c[k]).cuda()
    s = steps.HeadMlpStep(dev("Wemb"), dev("Wfc"), dev("Wproj"), T)
    X, dL = c["X"].cuda(), c["dLogits"].cuda()
    g = _capture(lambda st: s.step(X, dL, st))
    s.step(X, dL)
    torch.cuda.synchronize()
    Z0, logits0 = s.Z.clone(), s.logits.clone()
    outs = (s.Z, s.logits, s.dZ, s.dX, s.dWemb, s.dWfc, s.dWproj)
    qe = o.quantize_weight(c["Wemb"], 8)
    qf, qp = o.quantize_weight(c["Wfc"], 6), o.quantize_weight(c["Wproj"], 6)
    for seed in (9, 10):  # the second replay runs on new inputs copied into X and dL
        cc = c if seed == 9 else sy.head_mlp_case(T=T, seed=seed)
        X.copy_(cc["X"])
        dL.copy_(cc["dLogits"])
        for t in outs:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert qat.device_error() == 0
        if seed == 9:  # deterministic forward GEMMs: the direct call's bits
            assert np.array_equal(bits16(s.Z), bits16(Z0))
            assert np.array_equal(bits16(s.logits), bits16(logits0))
        ref = o.head_mlp_step(qe, qf, qp, cc["X"].float().numpy(), cc["dLogits"].float().numpy())
        for name, t in (("Z", s.Z), ("logits", s.logits), ("dZ", s.dZ), ("dX", s.dX),
                        ("dWemb", s.dWemb), ("dWfc", s.dWfc), ("dWproj", s.dWproj)):
            assert_close(t, ref[name], "%s (seed %d)" % (name, seed))
