"""Small single-kernel cases for profiler captures (ncu -k ... -c ...), next to
the benchmark that times the same kernels at full size.

    python profile_cases.py <case> [--T tokens]

Each case sets up its inputs, launches the named kernel a few times and exits.
Cases are sized so one capture stays small (a few hundred MB on the device)
while the operands still exceed L2 where the DRAM counters matter.
"""
import argparse
import sys

import numpy as np
import torch

from quantization_aware_tiny_b200 import export as qexport
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import steps
from quantization_aware_tiny_b200 import synthetic as sy


def logits_fwd(T):
    c = sy.head_mlp_case(T=1, seed=0)
    q = qat.quantize_weight(torch.from_numpy(c["Wemb"]).cuda(), 8)
    Z = sy.act_bf16(np.random.default_rng(1), T, 512, std=0.25).cuda()
    Y = torch.empty((T, 8192), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        qat.qat_linear_fwd(Z, Y, 8, qw=q)


def logits_fwd_fused(T):
    """The same logits GEMM from the fp32 tied head: the GEMM quantizes it in
    its producer (no workspace is passed, so the fused path is taken)."""
    c = sy.head_mlp_case(T=1, seed=0)
    W = torch.from_numpy(c["Wemb"]).cuda()
    Z = sy.act_bf16(np.random.default_rng(1), T, 512, std=0.25).cuda()
    Y = torch.empty((T, 8192), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        qat.qat_linear_fwd(Z, Y, 8, W=W)


def head_dw(T):
    c = sy.head_mlp_case(T=1, seed=0)
    Z = sy.act_bf16(np.random.default_rng(1), T, 512, std=0.25).cuda()
    dL = sy.act_bf16(np.random.default_rng(2), T, 8192, std=0.01).cuda()
    dW = torch.empty((8192, 512), dtype=torch.float32, device="cuda")
    for _ in range(3):
        qat.qat_linear_bwd(Z, dL, 8, dW=dW, N=8192, K=512)
    del c


def head_dx(T):
    c = sy.head_mlp_case(T=1, seed=0)
    q = qat.quantize_weight(torch.from_numpy(c["Wemb"]).cuda(), 8)
    dL = sy.act_bf16(np.random.default_rng(2), T, 8192, std=0.01).cuda()
    dX = torch.empty((T, 512), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        qat.qat_linear_bwd(None, dL, 8, qw=q, dX=dX)


def mlp_step(T):
    """The int6 ReLU^2 MLP 512-2048-512 forward and backward (6 GEMMs per pass)."""
    c = sy.head_mlp_case(T=1, seed=0)
    d, H = 512, 2048
    qf = qat.quantize_weight(torch.from_numpy(c["Wfc"]).cuda(), 6)
    qp = qat.quantize_weight(torch.from_numpy(c["Wproj"]).cuda(), 6)
    X = sy.act_bf16(np.random.default_rng(1), T, d).cuda()
    dY = sy.act_bf16(np.random.default_rng(2), T, d, std=0.01).cuda()
    bf = torch.bfloat16
    Y, dX = (torch.empty((T, d), dtype=bf, device="cuda") for _ in range(2))
    pre, h = (torch.empty((T, H), dtype=bf, device="cuda") for _ in range(2))
    dWfc = torch.empty((H, d), dtype=torch.float32, device="cuda")
    dWproj = torch.empty((d, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(qat.workspace_size(qat.QAT_OP_MLP_BWD, d, H, T, False), dtype=torch.uint8,
                     device="cuda")
    for _ in range(3):
        qat.qat_mlp_fwd(X, Y, 6, d, H, qfc=qf, qproj=qp, pre_save=pre, h_save=h)
        qat.qat_mlp_bwd(X, pre, h, dY, 6, d, H, qfc=qf, qproj=qp, dX=dX, dWfc=dWfc,
                        dWproj=dWproj, workspace=ws)


def export_state_dict(_T):
    sd = {k: torch.from_numpy(v).cuda() for k, v in sy.state_dict_case().items()}
    for _ in range(3):
        qexport.export_state_dict(sd)


def dequant_state_dict(_T):
    """The exported 11-layer state dict's int6 tensors back to fp32, one
    dequantize_rows_batch launch (after an export launch and an L2-sized
    write, so the codes start in DRAM)."""
    sd = {k: torch.from_numpy(v).cuda() for k, v in sy.state_dict_case().items()}
    ex = qexport.export_state_dict(sd)
    items = [(e["codes"], e["scale16"], torch.empty(e["codes"].shape, dtype=torch.float32, device="cuda"))
             for e in ex.values() if "codes" in e]
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for _ in range(3):
        flush.add_(1)
        qat.dequantize_rows_batch(items)


def quantize_step_weights(_T):
    """The training step's three weights (tied head 8192 x 512 int8, MLP fc
    2048 x 512 and proj 512 x 2048 int6) quantized to their bf16 operands in
    one qat_quantize_weights_batch launch, after a 256 MB write so the fp32
    weights start in DRAM."""
    c = sy.head_mlp_case(T=8)
    W = [torch.from_numpy(c[k]).cuda() for k in ("Wemb", "Wfc", "Wproj")]
    bits = (8, 6, 6)
    items = [(w, b, torch.empty(w.shape[0], dtype=torch.float32, device="cuda"), None,
              torch.empty(w.shape, dtype=torch.bfloat16, device="cuda")) for w, b in zip(W, bits)]
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for _ in range(3):
        flush.add_(1)
        qat.qat_quantize_weights_batch(items)


def core_train(T):
    """The d=640 recurrent core (R=3): forward keeping activations and the
    backward over the three applications (8 backward GEMMs per application)."""
    c = sy.recurrent_core_case(T=T)
    w = {k: torch.from_numpy(c[k]).cuda() for k in ("Wq", "Wk", "Wv", "Wo", "Wfc", "Wproj")}
    core = steps.RecurrentCore(w["Wq"], w["Wk"], w["Wv"], w["Wo"], w["Wfc"], w["Wproj"], 6)
    x = c["X"].cuda()
    dY = sy.act_bf16(np.random.default_rng(3), T, 640, std=0.01).cuda()
    for _ in range(2):
        core.forward_train(x, 3)
        core.backward(dY)


CASES = {"core_train": core_train, "logits_fwd": logits_fwd, "logits_fwd_fused": logits_fwd_fused, "head_dw": head_dw, "head_dx": head_dx,
         "mlp_step": mlp_step, "export_state_dict": export_state_dict, "dequant_state_dict": dequant_state_dict,
         "quantize_step_weights": quantize_step_weights}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--T", type=int, default=8192)
    a = ap.parse_args(argv)
    CASES[a.case](a.T)
    torch.cuda.synchronize()
    rc = qat.device_error()
    print("%s T=%d ok (device error %d)" % (a.case, a.T, rc))
    return rc


if __name__ == "__main__":
    sys.exit(main())
