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


def assert_close_chain(gpu, ref, roundings, what=""):
    """Chained bf16 state (the recurrent core): the state is re-rounded to bf16
    `roundings` times, and either side may land on the neighbouring bf16 value
    at each rounding -- an absolute change of one ulp of that element, at most
    2^-7 times the largest |state| of its row.  A residual add that cancels
    carries that absolute change into a small result, so on top of the
    single-op tolerance each element may differ by roundings * 2^-7 * row max."""
    g = np.asarray(to_np(gpu) if isinstance(gpu, torch.Tensor) else gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape and np.all(np.isfinite(g)), what
    fro = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    rowmax = np.max(np.abs(r), axis=1, keepdims=True)
    allow = ABS_REL * (np.abs(r) + 1.0) + roundings * 2.0 ** -7 * rowmax
    assert fro <= REL_FRO, "%s: relative Frobenius error %.3g" % (what, fro)
    assert np.all(np.abs(g - r) <= allow), "%s: max excess %.3g" % (what, np.max(np.abs(g - r) - allow))
    return fro
