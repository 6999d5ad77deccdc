"""Seeded synthetic inputs shaped like the record models' workloads.

This module holds random draws only -- none of the quantizer's or the GEMMs'
arithmetic -- so both the CUDA path's tests and the CPU oracle can take their
inputs from it.  numpy PCG64 streams spawned from SeedSequence(seed), one
child stream per tensor, in the order each function lists them.

Shapes follow the pages' models: d=512 with MLP 3x (1536) and 4x (2048),
8 query / 4 KV heads, tied vocab 1024 or 8192; the 3x3 recurrent core at
d=640 (head dim 80).  Weights are fp32 N(0, 0.02); activations are N(0, 1)
rounded to bf16; upstream gradients are N(0, 0.01) rounded to bf16.
"""
import numpy as np
import torch

W_STD = 0.02
DY_STD = 1e-2


def _streams(seed, n):
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(n)]


def weight(rng, rows, cols, std=W_STD):
    return (rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std))


def act_bf16(rng, rows, cols, std=1.0):
    """Gaussian activations as a CPU bf16 tensor."""
    a = rng.standard_normal((rows, cols), dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return torch.from_numpy(a).to(torch.bfloat16)


def with_outliers(rng, W, frac=1e-3, factor=20.0):
    """Multiply a seeded choice of frac*size entries by factor."""
    n = int(round(frac * W.size))
    idx = rng.choice(W.size, size=n, replace=False)
    flat = W.reshape(-1)
    flat[idx] *= np.float32(factor)
    return W


def heavy_tail_rows(rng, W, frac=0.05, nu=3.0, std=W_STD):
    """Replace a seeded choice of rows by std * Student-t(nu) draws."""
    rows = W.shape[0]
    n = max(1, int(round(frac * rows)))
    idx = rng.choice(rows, size=n, replace=False)
    W[idx] = (rng.standard_t(nu, size=(n, W.shape[1])) * std).astype(np.float32)
    return W


def linear_case(N=512, K=512, T=256, seed=0, outliers=True, with_dy=False):
    """Single CastedLinear: W [N,K] fp32 (0.1% entries x20), X [T,K] bf16."""
    r = _streams(seed, 4)
    W = weight(r[0], N, K)
    if outliers:
        with_outliers(r[1], W)
    X = act_bf16(r[2], T, K)
    out = {"W": W, "X": X}
    if with_dy:
        out["dY"] = act_bf16(r[3], T, N, DY_STD)
    return out


def mlp_case(d=512, H=1536, T=8192, seed=0):
    """ReLU^2 MLP block: Wfc [H,d], Wproj [d,H], X [T,d], dY [T,d]."""
    r = _streams(seed, 4)
    return {"Wfc": weight(r[0], H, d), "Wproj": weight(r[1], d, H),
            "X": act_bf16(r[2], T, d), "dY": act_bf16(r[3], T, d, DY_STD)}


def recurrent_core_case(d=640, H=1920, T=16384, seed=0):
    """3x3 core at d=640, 8 query / 4 KV heads of dim 80: Q [d,d], K,V [d/2,d],
    O [d,d], fc [H,d], proj [d,H]; X [T,d]."""
    r = _streams(seed, 7)
    return {"Wq": weight(r[0], d, d), "Wk": weight(r[1], d // 2, d),
            "Wv": weight(r[2], d // 2, d), "Wo": weight(r[3], d, d),
            "Wfc": weight(r[4], H, d), "Wproj": weight(r[5], d, H),
            "X": act_bf16(r[6], T, d)}


def head_mlp_case(T=4096, vocab=8192, d=512, H=2048, seed=0):
    """Tied head [vocab,d] + 4x MLP; X [T,d]; upstream dLogits [T,vocab]."""
    r = _streams(seed, 5)
    return {"Wemb": weight(r[0], vocab, d), "Wfc": weight(r[1], H, d),
            "Wproj": weight(r[2], d, H), "X": act_bf16(r[3], T, d),
            "dLogits": act_bf16(r[4], T, vocab, DY_STD)}


def state_dict_case(n_layers=11, d=512, mlp_mult=3, vocab=1024, seed=0):
    """11-layer d=512 state dict: per block Q, K, V, O, fc, proj (5% heavy-tailed
    rows each), per-block resid_mix [2,d], global skip_weights [5,d], tied
    embedding [vocab,d].  Returns an ordered dict name -> fp32 array."""
    names = []
    for i in range(n_layers):
        p = "blocks.%d." % i
        names += [(p + "attn.c_q.weight", d, d), (p + "attn.c_k.weight", d // 2, d),
                  (p + "attn.c_v.weight", d // 2, d), (p + "attn.proj.weight", d, d),
                  (p + "mlp.fc.weight", mlp_mult * d, d),
                  (p + "mlp.proj.weight", d, mlp_mult * d)]
    r = _streams(seed, 2 * len(names) + n_layers + 2)
    sd = {}
    k = 0
    for name, rows, cols in names:
        W = weight(r[k], rows, cols)
        heavy_tail_rows(r[k + 1], W)
        sd[name] = W
        k += 2
    for i in range(n_layers):
        sd["blocks.%d.resid_mix" % i] = weight(r[k], 2, d, std=1.0)
        k += 1
    sd["skip_weights"] = weight(r[k], 5, d, std=1.0)
    sd["tok_emb.weight"] = weight(r[k + 1], vocab, d)
    return sd
