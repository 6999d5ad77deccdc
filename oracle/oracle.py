"""Plain, slow, obviously correct CPU oracle (test infrastructure only).

Scalar quantizers come from qat_oracle.c through ctypes; the dense algebra is
numpy float64 on the exact values of the bf16 operands.  Nothing here is
blocked, fused or reordered beyond the definitions it restates.

Page references (title, section):
  P5 = "parameter-golf 16MB 极限压缩实战：11L MLP3x + Int6 QAT + zstd-22 记录详解"
  P1 = "Depth Recurrence + Mixed-Precision Quant" write-up (PR #363)
"""
import ctypes
import re

import numpy as np

from .build import build_oracle

# P5 "后训练量化导出": per-row clip at the 99.99984th percentile.
EXPORT_CLIP_Q = 0.9999984
# P5 "后训练量化导出": INT8_KEEP_FLOAT_MAX_NUMEL = 65_536 (reading: <= passes through).
KEEP_FLOAT_MAX_NUMEL = 65536

_lib = None


def _c():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_qat_scales.argtypes = [P, I64, I64, P]
        lib.oracle_qat_scales_bits.argtypes = [P, I64, I64, ctypes.c_int, P]
        lib.oracle_pack6.argtypes = [P, I64, ctypes.c_int, P]
        lib.oracle_export_rows_search.argtypes = [P, I64, I64, ctypes.c_int, P, ctypes.c_int,
                                                  P, P, P, P, P]
        lib.oracle_unpack6.argtypes = [P, I64, ctypes.c_int, P]
        lib.oracle_qat_codes.argtypes = [P, I64, I64, P, ctypes.c_int, P]
        lib.oracle_qat_codes.restype = ctypes.c_int
        lib.oracle_dequant_f32.argtypes = [P, P, I64, I64, P]
        lib.oracle_operand_bf16.argtypes = [P, P, I64, I64, P]
        lib.oracle_row_quantile_abs.argtypes = [P, I64, ctypes.c_double]
        lib.oracle_row_quantile_abs.restype = ctypes.c_float
        lib.oracle_export_rows.argtypes = [P, I64, I64, ctypes.c_int, ctypes.c_double, P, P, P]
        lib.oracle_export_rows.restype = ctypes.c_int
        lib.oracle_dequant_export.argtypes = [P, P, I64, I64, P]
        lib.oracle_fp16_array.argtypes = [P, I64, P]
        lib.oracle_bf16_array.argtypes = [P, I64, P]
        lib.oracle_philox4x32_10.argtypes = [P, P, P]
        lib.oracle_noisy_operand.argtypes = [P, I64, I64, ctypes.c_int, ctypes.c_uint64,
                                             ctypes.c_uint64, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- conversions

def bf16_bits(x):
    """bf16 round-to-nearest-even of fp32 values, as uint16 bit patterns."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint16)
    _c().oracle_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x):
    """Values of bf16_rne(x) as fp32."""
    return bf16_bits_to_f32(bf16_bits(x))


def fp16_bits(x):
    """binary16 round-to-nearest-even of fp32 values, as uint16 bit patterns."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint16)
    _c().oracle_fp16_array(_ptr(x), x.size, _ptr(out))
    return out


# ------------------------------------------------- QAT fake quantization (P5)

def qat_scales(W, bits=8):
    """P5 "训练时的模拟量化": s_i = max(max_j |W_ij|, 1e-12) / 127 (fp32); for
    bits = 5 the divisor is 15 (P1 "更多算力下…": the int5 step amax / 15)."""
    W = _f32(W)
    N, K = W.shape
    s = np.empty(N, np.float32)
    _c().oracle_qat_scales_bits(_ptr(W), N, K, int(bits), _ptr(s))
    return s


def qat_codes(W, scales, bits):
    """P5 "训练时的模拟量化": int6 c = clamp(4*rne(rne(w/s)/4), -128, 124);
    int8 c = clamp(rne(w/s), -127, 127); int5 c = clamp(rne(w/s), -15, 15)."""
    W = _f32(W)
    s = _f32(scales)
    N, K = W.shape
    c = np.empty((N, K), np.int8)
    rc = _c().oracle_qat_codes(_ptr(W), N, K, _ptr(s), int(bits), _ptr(c))
    if rc != 0:
        raise ValueError("bits must be 5, 6 or 8")
    return c


def dequant(codes, scales):
    """STE forward value Wq = fl32(c * s)."""
    c = np.ascontiguousarray(codes, np.int8)
    s = _f32(scales)
    N, K = c.shape
    out = np.empty((N, K), np.float32)
    _c().oracle_dequant_f32(_ptr(c), _ptr(s), N, K, _ptr(out))
    return out


def operand_bf16_bits(codes, scales):
    """GEMM operand bf16_rne(fl32(c * s)) as uint16 bits (P5: CastedLinear
    casts the quantized weight to the activation dtype)."""
    c = np.ascontiguousarray(codes, np.int8)
    s = _f32(scales)
    N, K = c.shape
    out = np.empty((N, K), np.uint16)
    _c().oracle_operand_bf16(_ptr(c), _ptr(s), N, K, _ptr(out))
    return out


def quantize_weight(W, bits):
    """Quantize once (also the recurrence cache: P1 "税 1", shared weights are
    stored once and quantized once).  Returns codes, scales, the fp32 STE
    value and the bf16 operand (as float64 for the algebra)."""
    s = qat_scales(W, bits)
    c = qat_codes(W, s, bits)
    op = bf16_bits_to_f32(operand_bf16_bits(c, s)).astype(np.float64)
    return {"codes": c, "scales": s, "wq": dequant(c, s), "operand": op}


# ------------------------------------------------ Noisy QAT (P1 "幸存发现 1")

def philox4x32_10(counter, key):
    """Philox-4x32-10 block (Salmon et al., SC'11) of a 4-word counter and a
    2-word key, as 4 uint32."""
    c = np.ascontiguousarray(counter, np.uint32)
    k = np.ascontiguousarray(key, np.uint32)
    out = np.empty(4, np.uint32)
    _c().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def noisy_weight(W, seed, offset=0, bits=8):
    """P1 "幸存发现 1 Noisy QAT": w + (u - 0.5) * max(amax,1e-12)/127 per row (the
    int8 step; bits = 5 uses the int5 step amax/15), u from Philox-4x32-10
    (counter = element // 4 and offset, key = seed).  Returns the fp32 scales,
    the noisy fp32 weight and its bf16 operand (float64 values)."""
    W = _f32(W)
    N, K = W.shape
    s = np.empty(N, np.float32)
    noisy = np.empty((N, K), np.float32)
    op = np.empty((N, K), np.uint16)
    _c().oracle_noisy_operand(_ptr(W), N, K, int(bits), int(seed), int(offset), _ptr(s),
                              _ptr(noisy), _ptr(op))
    return {"scales": s, "noisy": noisy, "operand_bits": op,
            "operand": bf16_bits_to_f32(op).astype(np.float64)}


# -------------------------------------------------------- dense algebra (fp64)

def _f64(x):
    return np.asarray(x, dtype=np.float64)


def linear_fwd(Wop, X):
    """P5 CastedLinear forward: Y = X . Wq^T (Wq the bf16 operand)."""
    return _f64(X) @ _f64(Wop).T


def linear_bwd(Wop, X, dY):
    """STE backward (P5 "训练时的模拟量化": the gradient w.r.t. the fp32 weight
    is the gradient w.r.t. the quantized weight): dX = dY . Wq, dW = dY^T . X."""
    dY = _f64(dY)
    return dY @ _f64(Wop), dY.T @ _f64(X)


def relu2(x):
    x = _f64(x)
    r = np.maximum(x, 0.0)
    return r * r


def leaky2(x):
    """LeakyReLU(0.5)^2 (P1 negative result #9; P4 leaderboard "LeakyReLU²")."""
    x = _f64(x)
    l = np.where(x > 0, x, 0.5 * x)
    return l * l


def mlp_fwd(Wfc_op, Wproj_op, X, act="relu2"):
    """P5 "架构": MLP(x) = proj(relu(fc(x))^2) (act = "leaky2": proj(leaky_relu(fc(x), 0.5)^2)).
    Returns pre, h, Y."""
    pre = _f64(X) @ _f64(Wfc_op).T
    h = relu2(pre) if act == "relu2" else leaky2(pre)
    return pre, h, h @ _f64(Wproj_op).T


def act_grad(pre, act="relu2"):
    """d(act(pre))/d(pre): relu^2 -> 2 relu(pre); leaky(0.5)^2 -> 2x (x>0), x/2 (x<0)."""
    pre = _f64(pre)
    if act == "relu2":
        return 2.0 * np.maximum(pre, 0.0)
    return np.where(pre > 0, 2.0 * pre, 0.5 * pre)


def mlp_bwd(Wfc_op, Wproj_op, X, pre, h, dY, act="relu2"):
    """Chain rule through proj, the activation (relu^2: derivative 2*relu(pre))
    and fc, with the STE making the quantized weights' gradients the weights'
    gradients."""
    dY = _f64(dY)
    dh = dY @ _f64(Wproj_op)
    dpre = dh * act_grad(pre, act)
    dWproj = dY.T @ _f64(h)
    dWfc = dpre.T @ _f64(X)
    dX = dpre @ _f64(Wfc_op)
    return dX, dWfc, dWproj


def _bf16_or_exact(exact):
    """The rounding applied where the core materialises an activation or a
    gradient tensor: bf16 round-to-nearest-even (the pages train in bf16), or
    none at all (exact=True: the plain fp64 composition, which the
    finite-difference pins differentiate)."""
    if exact:
        return lambda a: _f64(a)
    return lambda a: bf16_round(_f64(a).astype(np.float32)).astype(np.float64)


def core_application_fwd(ops, x, d, act="relu2", exact=False):
    """One application of the depth-recurrent core block (P1 "Stem / Core /
    Tail"; attention left out, so the O projection reads the query slice of
    QKV -- a reading stated in the design notes).  ops = (qkv, o, fc, proj),
    each a dict with the bf16 "operand" of that weight; x [T,d] is the state.
        qkv = x Wqkv^T ; x1 = x + q Wo^T ; pre = x1 Wfc^T ; h = act(pre)
        out = x1 + h Wproj^T
    Each tensor handed from one GEMM to the next (qkv, x1, pre, h, out) is
    rounded to bf16 once where it is materialised (exact=False); every sum and
    product in between is exact fp64.  Returns the saved activations
    {x, qkv, x1, pre, h, out} and the unrounded residual sums u1 (of x1) and
    u2 (of out)."""
    b = _bf16_or_exact(exact)
    q_qkv, q_o, q_fc, q_proj = ops
    x = _f64(x)
    qkv = b(x @ q_qkv["operand"].T)
    u1 = x + qkv[:, :d] @ q_o["operand"].T
    x1 = b(u1)
    pre_exact = x1 @ q_fc["operand"].T
    h = b(relu2(pre_exact) if act == "relu2" else leaky2(pre_exact))
    u2 = x1 + h @ q_proj["operand"].T
    return {"x": x, "qkv": qkv, "x1": x1, "pre": b(pre_exact), "h": h, "out": b(u2),
            "u1": u1, "u2": u2}


def core_fwd_apps(apps_ops, X, d, act="relu2", exact=False):
    """The core applied once per entry of apps_ops (application r uses
    apps_ops[r]); returns the final state and the list of saved activations."""
    x = _bf16_or_exact(exact)(_f64(X))
    saved = []
    for ops in apps_ops:
        s = core_application_fwd(ops, x, d, act, exact)
        saved.append(s)
        x = s["out"]
    return x, saved


def recurrent_core_fwd(q_qkv, q_o, q_fc, q_proj, X, R, d, act="relu2", exact=False):
    """Depth-recurrent core (P1 "Stem / Core / Tail", "税 1"): the block's
    linears, quantized once, applied R times (see core_application_fwd)."""
    return core_fwd_apps([(q_qkv, q_o, q_fc, q_proj)] * R, X, d, act, exact)[0]


def core_application_bwd(ops, s, g, d, act="relu2", exact=False):
    """Backward of one core application (chain rule through
    core_application_fwd, STE: the quantized weights' gradients are the fp32
    weights' gradients).  s = that application's saved activations, g = dL/d out.
        dWproj = g^T h ; dpre = (g Wproj) * act'(pre) ; dWfc = dpre^T x1
        dx1 = g + dpre Wfc            (residual of out = x1 + ...)
        dWo = dx1^T q ; dq = dx1 Wo
        dWqkv[:d] = dq^T x ; dWqkv[d:] = 0   (k and v do not reach the output
                                               with attention left out)
        dx = dx1 + dq Wq              (residual of x1 = x + ...)
    The gradient tensors handed between GEMMs (dpre, dx1, dq, dx) are rounded
    to bf16 where materialised (exact=False), as the forward's activations.
    Returns dx, the four weight gradients {qkv, o, fc, proj} and the
    intermediate gradients {dpre, dx1, dq}."""
    b = _bf16_or_exact(exact)
    q_qkv, q_o, q_fc, q_proj = ops
    g = _f64(g)
    dWproj = g.T @ s["h"]
    dpre = b((g @ q_proj["operand"]) * act_grad(s["pre"], act))
    dWfc = dpre.T @ s["x1"]
    dx1 = b(g + dpre @ q_fc["operand"])
    q = s["qkv"][:, :d]
    dWo = dx1.T @ q
    dq = b(dx1 @ q_o["operand"])
    dWqkv = np.zeros(q_qkv["operand"].shape)
    dWqkv[:d] = dq.T @ s["x"]
    dx = b(dx1 + dq @ q_qkv["operand"][:d])
    return dx, {"qkv": dWqkv, "o": dWo, "fc": dWfc, "proj": dWproj}, \
        {"dpre": dpre, "dx1": dx1, "dq": dq}


def core_bwd_apps(apps_ops, saved, dY, d, act="relu2", exact=False):
    """Backward through the applications in reverse order; each shared weight's
    gradient is the sum of its gradients over the applications that used it
    (P1 "税 1": one stored weight, R uses).  Returns dX, the four summed weight
    gradients, the incoming gradient of every application (grads[r] =
    dL/d out of application r) and each application's intermediate
    gradients."""
    g = _bf16_or_exact(exact)(_f64(dY))
    tot = None
    grads = [None] * len(saved)
    inter = [None] * len(saved)
    for r in reversed(range(len(saved))):
        grads[r] = g
        g, dW, inter[r] = core_application_bwd(apps_ops[r], saved[r], g, d, act, exact)
        tot = dW if tot is None else {k: tot[k] + dW[k] for k in tot}
    return g, tot, grads, inter


def recurrent_core_bwd(q_qkv, q_o, q_fc, q_proj, X, dY, R, d, act="relu2", exact=False):
    """Forward and STE backward of the recurrent core (quantized once, applied
    R times in the forward and R times, in reverse, in the backward, dW summed
    over the R uses).  dY = dL/d x_R.  Returns {out, dX, dWqkv, dWo, dWfc,
    dWproj, saved, grads}."""
    ops = [(q_qkv, q_o, q_fc, q_proj)] * R
    out, saved = core_fwd_apps(ops, X, d, act, exact)
    dX, dW, grads, inter = core_bwd_apps(ops, saved, dY, d, act, exact)
    return {"out": out, "dX": dX, "dWqkv": dW["qkv"], "dWo": dW["o"], "dWfc": dW["fc"],
            "dWproj": dW["proj"], "saved": saved, "grads": grads, "inter": inter}


def noisy_core_ops(Ws, R, seed, offset, bits=6):
    """Noisy QAT operands of the core (P1 "幸存发现 1"): application r draws the
    four weights (qkv, o, fc, proj -> k = 0..3) at Philox offset
    offset + 4*r + k (noise at the int8 step, or the int5 step for bits = 5)."""
    return [tuple({"operand": noisy_weight(w, seed, offset + 4 * r + k, bits)["operand"]}
                  for k, w in enumerate(Ws)) for r in range(R)]


def recurrent_core_fwd_noisy(Ws, X, R, d, seed, offset, bits=6, act="relu2"):
    """The recurrent core under Noisy QAT: application r uses its own noisy
    operands (noisy_core_ops), composed exactly as recurrent_core_fwd."""
    return core_fwd_apps(noisy_core_ops(Ws, R, seed, offset, bits), X, d, act)[0]


def recurrent_core_bwd_noisy(Ws, X, dY, R, d, seed, offset, bits=6, act="relu2"):
    """Forward and backward of the Noisy-QAT core: the backward of application
    r uses that application's noisy operands (the noise carries no gradient,
    so the weight gradient is the operand's)."""
    ops = noisy_core_ops(Ws, R, seed, offset, bits)
    out, saved = core_fwd_apps(ops, X, d, act)
    dX, dW, grads, inter = core_bwd_apps(ops, saved, dY, d, act)
    return {"out": out, "dX": dX, "dWqkv": dW["qkv"], "dWo": dW["o"], "dWfc": dW["fc"],
            "dWproj": dW["proj"], "saved": saved, "grads": grads, "inter": inter}


def head_mlp_step(q_emb, q_fc, q_proj, X, dLogits, act="relu2"):
    """Tied-head throughput step: Z = MLP(X), logits = Z Wemb^T, then the STE
    backward of both from the upstream gradient dLogits."""
    pre, h, Z = mlp_fwd(q_fc["operand"], q_proj["operand"], X, act)
    logits = Z @ q_emb["operand"].T
    dZ, dWemb = linear_bwd(q_emb["operand"], Z, dLogits)
    dX, dWfc, dWproj = mlp_bwd(q_fc["operand"], q_proj["operand"], X, pre, h, dZ, act)
    return {"pre": pre, "h": h, "Z": Z, "logits": logits, "dZ": dZ, "dWemb": dWemb,
            "dX": dX, "dWfc": dWfc, "dWproj": dWproj}


# ---------------------------------------------------------- export quantizer

def row_quantile_abs(row, q=EXPORT_CLIP_Q):
    """Linear-interpolated quantile of |row| (P5 "后训练量化导出")."""
    r = _f32(row)
    return float(_c().oracle_row_quantile_abs(_ptr(r), r.size, float(q)))


def export_rows(W, bits, q=EXPORT_CLIP_Q):
    """P5 "后训练量化导出": per-row clip, int6/int8 codes, fp16 scales.
    Returns codes (int8), fp16 scale bits (uint16), fp32 scales."""
    W = _f32(W)
    rows, cols = W.shape
    c = np.empty((rows, cols), np.int8)
    s16 = np.empty(rows, np.uint16)
    s32 = np.empty(rows, np.float32)
    rc = _c().oracle_export_rows(_ptr(W), rows, cols, int(bits), float(q), _ptr(c),
                                 _ptr(s16), _ptr(s32))
    if rc != 0:
        raise ValueError("bits must be 5, 6 or 8")
    return c, s16, s32


# Clip-search candidates (reading of "GPTQ-lite 裁剪搜索"; the pages give no
# list): the row maximum, the export's own 99.99984 percentile, then four
# tighter clips; the first of equal errors (the widest clip) is kept.
CLIP_CANDIDATES = (1.0, 0.9999984, 0.99999, 0.9999, 0.9995, 0.999)


def export_rows_search(W, bits, cand=CLIP_CANDIDATES):
    """P4 leaderboard "GPTQ-lite 裁剪搜索" (undefined there): per row, export at
    every candidate clip quantile and keep the one whose stored row (codes times
    the fp16 scale) has the least squared error against w.  Returns codes,
    fp16 scale bits, fp32 scales, the kept candidate index per row and the
    errors [rows, len(cand)]."""
    W = _f32(W)
    rows, cols = W.shape
    cd = np.ascontiguousarray(cand, np.float64)
    c = np.empty((rows, cols), np.int8)
    s16 = np.empty(rows, np.uint16)
    s32 = np.empty(rows, np.float32)
    ch = np.empty(rows, np.int32)
    errs = np.empty((rows, cd.size), np.float64)
    rc = _c().oracle_export_rows_search(_ptr(W), rows, cols, int(bits), _ptr(cd), cd.size,
                                        _ptr(c), _ptr(s16), _ptr(s32), _ptr(ch), _ptr(errs))
    if rc != 0:
        raise ValueError("bits must be 5, 6 or 8")
    return c, s16, s32, ch, errs


def dequant_export(codes, scale16_bits):
    """Roundtrip dequantize: fl32(c * fp32(fp16 scale))."""
    c = np.ascontiguousarray(codes, np.int8)
    s = np.ascontiguousarray(scale16_bits, np.uint16)
    rows, cols = c.shape
    out = np.empty((rows, cols), np.float32)
    _c().oracle_dequant_export(_ptr(c), _ptr(s), rows, cols, _ptr(out))
    return out


def pack6(codes, bits):
    """6-bit packing of int6 / int5 codes (P1 Day 0 "bit-packing"): field c/4
    (int6) or c (int5), 6 bits two's complement, little-endian bit stream,
    4 codes -> 3 bytes.  Returns uint8 [3*n/4] for the flattened codes."""
    c = np.ascontiguousarray(codes, np.int8).reshape(-1)
    out = np.empty(3 * c.size // 4, np.uint8)
    if _c().oracle_pack6(_ptr(c), c.size, int(bits), _ptr(out)) != 0:
        raise ValueError("pack6 needs bits 5 or 6 and a multiple of 4 codes")
    return out


def unpack6(packed, n, bits):
    """Inverse of pack6: n int8 codes."""
    p = np.ascontiguousarray(packed, np.uint8).reshape(-1)
    out = np.empty(n, np.int8)
    if _c().oracle_unpack6(_ptr(p), n, int(bits), _ptr(out)) != 0:
        raise ValueError("unpack6 needs bits 5 or 6 and a multiple of 4 codes")
    return out


_BLOCK_RE = re.compile(r"^blocks\.(\d+)\.")


def export_state_dict(sd, int6_start=0, int6_end=10, fp16_embed_name="tok_emb.weight",
                      keep_float_max=KEEP_FLOAT_MAX_NUMEL, mlp_int5=False, attn_int5=False):
    """P5 "后训练量化导出" rules, tensor by tensor:
    non-2D or numel <= keep_float_max -> fp16 passthrough; the tied embedding
    -> fp16 passthrough; other 2D tensors -> per-row codes, int6 when the
    tensor belongs to block i with int6_start <= i <= int6_end (inclusive,
    -1 switches int6 off), else int8.
    P1 reproduction commands (MLP_INT5 / ATTN_INT5): with mlp_int5 every block
    MLP weight ("blocks.<i>.mlp."), with attn_int5 every block attention weight
    ("blocks.<i>.attn.") is exported int5 instead (the mixed int5/int6 export)."""
    out = {}
    for name, t in sd.items():
        t = _f32(t)
        if t.ndim != 2 or t.size <= keep_float_max or name == fp16_embed_name:
            out[name] = {"kind": "fp16", "bits16": fp16_bits(t)}
            continue
        m = _BLOCK_RE.match(name)
        bits = 8
        if m and int6_start >= 0 and int6_end >= 0:
            i = int(m.group(1))
            if int6_start <= i <= int6_end:
                bits = 6
        if m and ((mlp_int5 and ".mlp." in name) or (attn_int5 and ".attn." in name)):
            bits = 5
        c, s16, _ = export_rows(t, bits)
        out[name] = {"kind": "int%d" % bits, "codes": c, "scale16": s16}
    return out
