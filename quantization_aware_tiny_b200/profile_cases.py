"""Small single-kernel cases for profiler captures (ncu -k ... -c ...).

    python -m quantization_aware_tiny_b200.profile_cases <case> [--T tokens]

Each case sets up its inputs, launches the named kernel a few times and exits.
Cases are sized so one capture stays small (a few hundred MB on the device)
while the operands still exceed L2 where the DRAM counters matter.
"""
import argparse
import sys

import numpy as np
import torch

from . import export as qexport
from . import qat
from . import synthetic as sy


def logits_fwd(T):
    c = sy.head_mlp_case(T=1, seed=0)
    q = qat.quantize_weight(torch.from_numpy(c["Wemb"]).cuda(), 8)
    Z = sy.act_bf16(np.random.default_rng(1), T, 512, std=0.25).cuda()
    Y = torch.empty((T, 8192), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        qat.qat_linear_fwd(Z, Y, 8, qw=q)


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


def export_state_dict(_T):
    sd = {k: torch.from_numpy(v).cuda() for k, v in sy.state_dict_case().items()}
    for _ in range(3):
        qexport.export_state_dict(sd)


CASES = {"logits_fwd": logits_fwd, "head_dw": head_dw, "head_dx": head_dx,
         "export_state_dict": export_state_dict}


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
