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


def bf16_ulp(v):
    """Spacing of bf16 values in the binade of |v| (8 significant bits); the
    smallest normal spacing below 2^-126."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7.0)


def chain_allowance(sums, factor=2.0):
    """Per-element allowance, on top of the single-op tolerance, for a state
    carried through a chain of residual adds that are each rounded to bf16
    (the recurrent core: x1 = bf16(x + o), out = bf16(x1 + m), twice per
    application).  `sums` are the oracle's unrounded residual sums in chain
    order, one array per rounding.

    Both sides round at the same points but their unrounded values differ
    slightly (the GPU accumulates in fp32, in its own order), so at each
    rounding either side may land on the neighbouring bf16 value: one ulp of
    the element's own magnitude there, ulp(|u_k| + A_{k-1}), carried on
    unchanged by the residual add.  The GEMM term of each add carries the
    neighbouring elements' flips in as well (one flipped element of q moves
    the whole row's q Wo^T; by the third application most of a row's h
    elements differ between the two sides); that part is allowed as the same
    size again: factor 2.  Measured: the largest excess over the single-op
    tolerance reaches 0.97 of the plain ulp sum in CPU emulations of other
    fp32 accumulation orders, and just over it on the B200."""
    A = np.zeros_like(np.asarray(sums[0], np.float64))
    for u in sums:
        A = A + bf16_ulp(np.abs(u) + factor * A)
    return factor * A


def core_sums(saved):
    """The residual sums of an oracle core run in chain order (u1, u2 of each
    application), for chain_allowance."""
    out = []
    for s in saved:
        out += [s["u1"], s["u2"]]
    return out


def rounding_noise_allowance(rounded, exact, z=6.0):
    """Element allowance, on top of the single-op tolerance, for a weight
    gradient summed over a chained core's tokens and applications.  Through
    the chain the two sides' bf16 rounding decisions decorrelate (most
    activation and gradient elements land on different neighbours), so their
    gradients differ like two independent draws of the chain's bf16 rounding
    noise.  The oracle measures that noise itself: the difference between its
    rounded run and its exact (unrounded) run, whose RMS over the tensor is
    sigma; two independent draws differ by sqrt(2) sigma, allowed at z
    standard deviations."""
    d = np.asarray(rounded, np.float64) - np.asarray(exact, np.float64)
    return z * np.sqrt(2.0) * np.sqrt(np.mean(d * d))


def assert_close_chain(gpu, ref, extra, what=""):
    """The single-op tolerance (relative Frobenius <= 5e-3, max excess over
    1e-2 * (|ref| + 1)) plus, element by element, the chain allowance
    `extra` (core_fwd_allowance / core_bwd_allowance)."""
    g = np.asarray(to_np(gpu) if isinstance(gpu, torch.Tensor) else gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape and np.all(np.isfinite(g)), what
    fro = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    allow = ABS_REL * (np.abs(r) + 1.0) + extra
    assert fro <= REL_FRO, "%s: relative Frobenius error %.3g" % (what, fro)
    bad = np.abs(g - r) > allow
    if np.any(bad):
        i = np.unravel_index(np.argmax(np.abs(g - r) - allow), g.shape)
        raise AssertionError("%s: %d elements beyond the allowance; worst at %s: gpu %.6g ref %.6g "
                             "tol %.3g chain %.3g" % (what, int(bad.sum()), i, g[i], r[i],
                                                      ABS_REL * (abs(r[i]) + 1), np.asarray(extra)[i]
                                                      if np.ndim(extra) else extra))
    return fro
