"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""
import numpy as np
import torch

# Floating-point outputs and gradients against the fp64 oracle:
# relative Frobenius error <= 5e-3 and max |err| <= 1e-2 * (|ref| + 1).
REL_FRO = 5e-3
ABS_REL = 1e-2


def to_np(t):
    t = t.detach()
    if t.dtype == torch.bfloat16 or t.dtype == torch.float16:
        t = t.float()
    return t.cpu().numpy()


def assert_close(gpu, ref, what=""):
    g = np.asarray(to_np(gpu) if isinstance(gpu, torch.Tensor) else gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what
    den = np.linalg.norm(r)
    fro = np.linalg.norm(g - r) / (den if den > 0 else 1.0)
    worst = np.max(np.abs(g - r) - ABS_REL * (np.abs(r) + 1.0)) if r.size else -1
    assert fro <= REL_FRO, "%s: relative Frobenius error %.3g" % (what, fro)
    assert worst <= 0, "%s: max elementwise excess %.3g" % (what, worst)
    return fro


def bits16(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
