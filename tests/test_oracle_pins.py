"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-derived example, a closed-form invariant, brute force on tiny inputs,
finite differences, or an independent library routine (numpy / torch IEEE
conversions, numpy.quantile).  Page references:
  P5 = "parameter-golf 16MB 极限压缩实战：11L MLP3x + Int6 QAT + zstd-22 记录详解"
  P1 = "Depth Recurrence + Mixed-Precision Quant" write-up (PR #363)
"""
import os

import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import synthetic as sy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = v.split()
    return d


# --------------------------------------------------------------- QAT codes

def test_worked_example_int6_int8():
    """P5 "训练时的模拟量化": hand-derived codes (ties to even at every .5)."""
    g = _golden("qat_worked_example.txt")
    W = np.array([g["w"]], dtype=np.float32)
    s = o.qat_scales(W)
    assert s[0] == np.float32(g["scale"][0])
    assert o.qat_codes(W, s, 6)[0].tolist() == [int(v) for v in g["int6"]]
    assert o.qat_codes(W, s, 8)[0].tolist() == [int(v) for v in g["int8"]]


def test_int5_worked_example():
    """P1 "幸存发现 1 Noisy QAT" (int5 step amax / 15) and the MLP_INT5 /
    ATTN_INT5 switches: hand-derived codes, ties to even."""
    g = _golden("int5_worked_example.txt")
    for r in ("W", "V"):
        W = np.array([g[r]], dtype=np.float32)
        s = o.qat_scales(W, 5)
        assert s[0] == np.float32(g[r + "_scale"][0])
        assert o.qat_codes(W, s, 5)[0].tolist() == [int(v) for v in g[r + "_int5"]]
    A = np.array([g["A"]], np.float32)
    c5, s16, _ = o.export_rows(A, 5)
    assert c5[0].tolist() == [int(v) for v in g["A_int5"]]
    assert int(s16[0]) == int(g["A_scale16"][0])


@pytest.mark.parametrize("seed", [0, 1])
def test_int5_grid_and_error_bound(seed):
    """int5: s = fl32(amax/15) (numpy IEEE division), codes in [-15, 15], the
    code is numpy's rne of the IEEE quotient, |w - c*s| <= s/2 (+ fp32
    roundings), and every row's amax element saturates to +-15."""
    W = sy.linear_case(seed=seed)["W"]
    s = o.qat_scales(W, 5)
    amax = np.abs(W).max(axis=1)
    assert np.array_equal(s, amax / np.float32(15.0))
    c = o.qat_codes(W, s, 5).astype(np.int32)
    assert c.min() >= -15 and c.max() <= 15
    assert np.array_equal(c, np.clip(np.rint(W / s[:, None]), -15, 15).astype(np.int32))
    err = np.abs(W.astype(np.float64) - o.dequant(c.astype(np.int8), s).astype(np.float64))
    assert np.all(err / s[:, None].astype(np.float64) <= 0.5 + 64 * 2.0 ** -24)
    im = np.argmax(np.abs(W), axis=1)
    cm = c[np.arange(W.shape[0]), im]
    assert np.array_equal(np.abs(cm), np.full(W.shape[0], 15))
    wq = o.dequant(c.astype(np.int8), s)
    assert np.array_equal(o.qat_codes(wq, s, 5), c.astype(np.int8))


def test_scale_is_ieee_division_and_floor():
    """s = fl32(max(amax, 1e-12) / 127) -- numpy float32 division is IEEE."""
    c = sy.linear_case()
    W = c["W"]
    s = o.qat_scales(W)
    amax = np.abs(W).max(axis=1)
    assert np.array_equal(s, amax / np.float32(127.0))
    Z = np.zeros((3, 40), np.float32)
    Z[1, 5] = 1e-20
    sz = o.qat_scales(Z)
    assert np.all(sz == np.float32(1e-12) / np.float32(127.0))
    assert np.all(o.qat_codes(Z, sz, 6) == 0)


@pytest.mark.parametrize("seed", [0, 1])
def test_codes_grid_and_integer_error(seed):
    """Codes are multiples of 4 in [-128,124], at most 64 distinct values, and
    |rne(w/s) - c| <= 2 wherever the clamp did not bind (closed form of
    double rounding)."""
    W = sy.linear_case(seed=seed)["W"]
    s = o.qat_scales(W)
    c = o.qat_codes(W, s, 6).astype(np.int32)
    assert c.min() >= -128 and c.max() <= 124
    assert np.all(c % 4 == 0)
    assert len(np.unique(c)) <= 64
    q_raw = np.rint(W / s[:, None])  # numpy IEEE float32 division + rint (half-even)
    unclamped = (q_raw <= 125) & (q_raw >= -126)
    assert np.all(np.abs(q_raw - c)[unclamped] <= 2)
    # positive row maxima always saturate to 124 (127 -> 31.75 -> 32 -> 128 -> 124)
    imax = np.argmax(W, axis=1)
    pos = W[np.arange(W.shape[0]), imax] == np.abs(W).max(axis=1)
    assert np.all(c[np.arange(W.shape[0]), imax][pos] == 124)


def test_error_bound_is_2p5_scale():
    """|w - c*s| <= (2.5 + 256*2^-24)*s unclamped and (3 + 256*2^-24)*s under
    positive saturation (the 2^-24 terms are the fp32 roundings of w/s, of s
    and of c*s).
    The 2*s bound quoted for this grid does not hold under double rounding:
    w/s = 2.4 -> 2 -> 0.5 -> 0 gives an error of 2.4*s."""
    W = sy.linear_case(N=512, K=512, seed=3)["W"]
    s = o.qat_scales(W)
    c = o.qat_codes(W, s, 6)
    wq = o.dequant(c, s).astype(np.float64)
    err = np.abs(W.astype(np.float64) - wq) / s[:, None].astype(np.float64)
    q_raw = np.rint(W / s[:, None])
    unclamped = (q_raw <= 125) & (q_raw >= -126)
    slack = 256 * 2.0 ** -24
    assert err[unclamped].max() <= 2.5 + slack
    assert err.max() <= 3.0 + slack
    assert (err[unclamped] > 2.0).any()
    one = np.array([[127.0, 2.4]], np.float32)
    assert o.qat_codes(one, o.qat_scales(one), 6)[0, 1] == 0


def test_fixed_scale_idempotence():
    """quant(fl32(c*s); s) == c, and dequant o quant o dequant == dequant."""
    W = sy.linear_case(seed=5)["W"]
    s = o.qat_scales(W)
    for bits in (6, 8):
        c = o.qat_codes(W, s, bits)
        wq = o.dequant(c, s)
        c2 = o.qat_codes(wq, s, bits)
        assert np.array_equal(c, c2)
        assert np.array_equal(o.dequant(c2, s), wq)


def test_rederived_scale_is_not_idempotent():
    """Re-deriving the scale from the dequantized row moves codes: row
    [127, 100] -> codes [124, 100] -> amax' = 124 -> 100/(124/127) = 102.4
    -> 102 -> 25.5 -> 26 -> 104."""
    W = np.array([[127.0, 100.0]], np.float32)
    c = o.qat_codes(W, o.qat_scales(W), 6)
    assert c[0].tolist() == [124, 100]
    wq = o.dequant(c, o.qat_scales(W))
    assert o.qat_codes(wq, o.qat_scales(wq), 6)[0].tolist() == [124, 104]


def test_operand_is_bf16_of_ste_value():
    """The STE forward operand equals the quantized weight cast to bf16
    (torch's rounding as the independent routine), and the cache's operand
    equals a fresh quantization (recurrence cache parity)."""
    W = sy.linear_case(seed=2)["W"]
    q = o.quantize_weight(W, 6)
    ref = torch.from_numpy(q["wq"]).to(torch.bfloat16).float().numpy()
    assert np.array_equal(q["operand"].astype(np.float32), ref)
    q2 = o.quantize_weight(W.copy(), 6)
    assert np.array_equal(q["codes"], q2["codes"]) and np.array_equal(q["operand"], q2["operand"])


def test_gqa_concat_quantization_is_exact():
    """Per-row quantization is per output row, so quantizing [Wq;Wk;Wv]
    together equals quantizing each and concatenating."""
    c = sy.recurrent_core_case(T=8)
    cat = np.concatenate([c["Wq"], c["Wk"], c["Wv"]], axis=0)
    qc = o.quantize_weight(cat, 6)
    parts = [o.quantize_weight(c[k], 6) for k in ("Wq", "Wk", "Wv")]
    assert np.array_equal(qc["codes"], np.concatenate([p["codes"] for p in parts]))
    assert np.array_equal(qc["scales"], np.concatenate([p["scales"] for p in parts]))


# -------------------------------------------------------------- conversions

def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32),
        # exact ties: low 16 bits == 0x8000 with both parities of the kept bit
        (np.arange(2000, dtype=np.uint32) << 16 | 0x8000 | 0x3f800000).view(np.float32),
        np.array([0.0, -0.0, 3.0e38, -3.0e38, 1e-45], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.bf16_bits(x), ref)


def test_fp16_rne_matches_numpy():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(50000).astype(np.float32) * (np.float32(2.0) ** rng.integers(-30, 18, 50000).astype(np.float32)),
        np.arange(-2048, 2048, dtype=np.float32) * np.float32(2.0 ** -25),  # subnormal ties
        np.array([65504.0, 65519.0, 65520.0, 1e6, -1e6, 0.0, -0.0, 6.1035156e-05,
                  6.097555e-05, 2.9802322e-08, 2.9802326e-08, 1.0009766, 1.0004883], np.float32)])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(o.fp16_bits(x), ref)


# -------------------------------------------------------------- quantile

def test_quantile_brute_force_tiny_rows():
    """P5 "后训练量化导出": sorted brute force on n = 2..17, random and tied rows.
    clip lies in [v_(n-2), v_(n-1)], equals v_lo when the top two tie, and
    agrees with numpy.quantile(method='linear') to 1 fp32 ulp."""
    rng = np.random.default_rng(7)
    for n in range(2, 18):
        for trial in range(40):
            row = rng.standard_normal(n).astype(np.float32)
            if trial % 4 == 0:
                row[rng.integers(n)] = -row[np.argmax(np.abs(row))]
            if trial % 4 == 1:
                row[:] = np.float32(rng.integers(-3, 4, n))
            v = np.sort(np.abs(row))
            clip = np.float32(o.row_quantile_abs(row))
            assert v[n - 2] <= clip <= v[n - 1]
            if v[n - 2] == v[n - 1]:
                assert clip == v[n - 1]
            ref = np.float32(np.quantile(np.abs(row).astype(np.float64), o.EXPORT_CLIP_Q))
            assert abs(float(clip) - float(ref)) <= float(np.spacing(np.float32(max(abs(ref), 1e-30))))


@pytest.mark.parametrize("n,frac", [(512, 0.9991824), (1536, 0.997544), (8192, 0.9868944)])
def test_quantile_fraction_closed_form(n, frac):
    """With top two |w| = 0 and 1 the clip equals the interpolation fraction
    1 - (1-q)(n-1) (position q(n-1) lands between the last two)."""
    row = np.zeros(n, np.float32)
    row[n // 3] = -1.0
    assert abs(o.row_quantile_abs(row) - frac) <= 1e-6
    assert abs(frac - (1 - 1.6e-6 * (n - 1))) < 1e-9


def test_export_worked_examples():
    g = _golden("export_worked_examples.txt")
    A = np.array([g["A"]], np.float32)
    c6, s16, s32 = o.export_rows(A, 6)
    assert c6[0].tolist() == [int(v) for v in g["A_int6"]]
    assert int(s16[0]) == int(g["A_scale16"][0]) and s32[0] == 1.0
    assert o.export_rows(A, 8)[0][0].tolist() == [int(v) for v in g["A_int8"]]
    B = np.array([g["B"]], np.float32)
    c6, s16, s32 = o.export_rows(B, 6)
    assert c6[0].tolist() == [int(v) for v in g["B_int6"]]
    assert int(s16[0]) == int(g["B_scale16"][0])
    assert abs(o.row_quantile_abs(B[0]) - float(g["B_clip"][0])) < 1e-4


def test_export_invariants_and_scale_encoding():
    """Export of heavy-tailed rows: s32 = max(clip,1e-12)/127 (numpy IEEE
    division), stored scale = fp16_rne(s32) (numpy conversion), codes on the
    grid with |clamp(w) - c*s32| <= 2.5*s32 unclamped, dequant = c*fp32(s16)."""
    sd = sy.state_dict_case(n_layers=1)
    W = sd["blocks.0.mlp.fc.weight"][:96]
    for bits in (6, 8):
        c, s16, s32 = o.export_rows(W, bits)
        clip = np.array([o.row_quantile_abs(r) for r in W], np.float32)
        assert np.array_equal(s32, np.maximum(clip, np.float32(1e-12)) / np.float32(127.0))
        assert np.array_equal(s16, s32.astype(np.float16).view(np.uint16))
        assert np.all(np.abs(W) .max(axis=1) >= clip)
        if bits == 6:
            assert np.all(c.astype(np.int32) % 4 == 0) and c.min() >= -128 and c.max() <= 124
        else:
            assert c.min() >= -127 and c.max() <= 127
        wc = np.clip(W, -clip[:, None], clip[:, None]).astype(np.float64)
        err = np.abs(wc - c.astype(np.float64) * s32[:, None]) / s32[:, None]
        lim = 2.5 if bits == 6 else 0.5
        inner = np.abs(wc) < clip[:, None] * (124.0 / 127.0 if bits == 6 else 1.0)
        assert err[inner].max() <= lim * (1 + 2.0 ** -20)
        deq = o.dequant_export(c, s16)
        ref = c.astype(np.float32) * s16.view(np.float16).astype(np.float32)[:, None]
        assert np.array_equal(deq, ref)


def test_export_passthrough_and_layer_range():
    """P5 "后训练量化导出": non-2D and small (<= 65,536 elements, reading of
    INT8_KEEP_FLOAT_MAX_NUMEL) tensors and the tied embedding pass through as
    fp16; blocks 0..10 inclusive are int6 (INT6_LAYER_START/END = 0/10), -1
    switches int6 off."""
    rng = np.random.default_rng(3)
    sd = {"blocks.0.a": rng.standard_normal((256, 256)).astype(np.float32),  # 65,536: passthrough
          "blocks.0.b": rng.standard_normal((300, 256)).astype(np.float32),
          "blocks.10.b": rng.standard_normal((300, 256)).astype(np.float32),
          "blocks.11.b": rng.standard_normal((300, 256)).astype(np.float32),
          "other": rng.standard_normal((1, 65537)).astype(np.float32),
          "vec": rng.standard_normal(100000).astype(np.float32),
          "tok_emb.weight": rng.standard_normal((1024, 512)).astype(np.float32)}
    out = o.export_state_dict(sd)
    kinds = {k: v["kind"] for k, v in out.items()}
    assert kinds == {"blocks.0.a": "fp16", "blocks.0.b": "int6", "blocks.10.b": "int6",
                     "blocks.11.b": "int8", "other": "int8", "vec": "fp16",
                     "tok_emb.weight": "fp16"}
    off = o.export_state_dict(sd, int6_start=-1, int6_end=-1)
    assert off["blocks.0.b"]["kind"] == "int8"
    sd5 = {"blocks.1.mlp.fc.weight": sd["blocks.0.b"], "blocks.12.attn.c_q.weight": sd["blocks.0.b"],
           "blocks.1.attn.c_q.weight": sd["blocks.0.b"]}
    k5 = {k: v["kind"] for k, v in o.export_state_dict(sd5, mlp_int5=True).items()}
    assert k5 == {"blocks.1.mlp.fc.weight": "int5", "blocks.12.attn.c_q.weight": "int8",
                  "blocks.1.attn.c_q.weight": "int6"}
    k5 = {k: v["kind"] for k, v in o.export_state_dict(sd5, mlp_int5=True, attn_int5=True).items()}
    assert set(k5.values()) == {"int5"}
    assert np.array_equal(out["vec"]["bits16"], sd["vec"].astype(np.float16).view(np.uint16))


def test_pack6_worked_example():
    """P1 Day 0 bit-packing, read as 6-bit little-endian fields: hand-derived bytes."""
    g = _golden("pack6_worked_example.txt")
    for bits in (6, 5):
        c = np.array([int(v) for v in g["int%d_codes" % bits]], np.int8)
        assert o.pack6(c, bits).tolist() == [int(v) for v in g["int%d_bytes" % bits]]


@pytest.mark.parametrize("bits", [5, 6])
def test_pack6_against_numpy_packbits_and_roundtrip(bits):
    """The packed stream equals numpy.packbits (little bit order) of the
    fields' bits; unpack inverts pack on every code of the grid and on export
    codes of a real row set; 4 codes take 3 bytes."""
    grid = np.arange(-128, 125, 4) if bits == 6 else np.arange(-15, 16)
    rng = np.random.default_rng(bits)
    c = rng.choice(grid, 4096).astype(np.int8)
    c[:len(grid)] = grid
    f = (c.astype(np.int32) // (4 if bits == 6 else 1)) & 63
    bitstream = ((f[:, None] >> np.arange(6)[None, :]) & 1).astype(np.uint8).reshape(-1)
    ref = np.packbits(bitstream, bitorder="little")
    p = o.pack6(c, bits)
    assert p.size == 3 * c.size // 4
    assert np.array_equal(p, ref)
    assert np.array_equal(o.unpack6(p, c.size, bits), c)
    W = sy.linear_case(N=64, K=256, seed=9)["W"]
    ce, _, _ = o.export_rows(W, bits)
    assert np.array_equal(o.unpack6(o.pack6(ce, bits), ce.size, bits).reshape(ce.shape), ce)


def _exact_err(w, c, s16):
    from fractions import Fraction
    sh = Fraction(float(np.uint16(s16).view(np.float16)))
    return sum((Fraction(float(x)) - int(k) * sh) ** 2 for x, k in zip(w, c))


@pytest.mark.parametrize("bits", [5, 6, 8])
def test_clip_search_minimises_exact_error(bits):
    """The clip search keeps, per row, the candidate whose stored row has the
    least squared error, checked with exact rational arithmetic on codes and
    scales produced by the plain export at each candidate quantile; the kept
    codes and scale are that export's."""
    sd = sy.state_dict_case(n_layers=1, seed=3)
    W = np.concatenate([sd["blocks.0.mlp.fc.weight"][:6], sd["blocks.0.mlp.proj.weight"][:3, :512]])
    W = np.ascontiguousarray(W)
    c, s16, s32, ch, errs = o.export_rows_search(W, bits)
    for i in range(W.shape[0]):
        exact = []
        for q in o.CLIP_CANDIDATES:
            ck, hk, _ = o.export_rows(W[i:i + 1], bits, q=q)
            exact.append(_exact_err(W[i], ck[0], hk[0]))
        best = min(exact)
        k = ch[i]
        assert exact[k] == best or float(exact[k] - best) <= 1e-12 * float(best), (i, k)
        assert all(e > exact[k] or j >= k for j, e in enumerate(exact) if e == exact[k])
        for j, e in enumerate(exact):
            assert abs(errs[i, j] - float(e)) <= 1e-9 * float(e) + 1e-30
        ck, hk, sk = o.export_rows(W[i:i + 1], bits, q=o.CLIP_CANDIDATES[k])
        assert np.array_equal(c[i], ck[0]) and s16[i] == hk[0] and s32[i] == sk[0]
    assert np.all(errs[np.arange(len(ch)), ch] <= errs[:, 1])   # never worse than the plain export


def test_clip_search_exact_row_and_outlier_row():
    """A row already on the int8 grid with a power-of-two scale keeps the row
    maximum at zero error; a row with one 10-sigma outlier gives up part of
    it for a finer grid on the rest when the grid is coarse (int5: a tight
    candidate wins by a wide margin)."""
    on_grid = np.array([np.arange(-127, 129, 2)[:128]], np.float32)   # amax 127 -> s = 1
    on_grid[0, 0] = 127.0
    c, s16, _, ch, errs = o.export_rows_search(on_grid, 8)
    assert ch[0] == 0 and errs[0, 0] == 0.0
    assert np.array_equal(c[0].astype(np.float32), on_grid[0])
    rng = np.random.default_rng(4)
    row = (rng.standard_normal((1, 4096)) * 0.01).astype(np.float32)
    row[0, 7] = 0.1
    _, _, _, ch, errs = o.export_rows_search(row, 5)
    assert ch[0] >= 3 and errs[0, ch[0]] < 0.5 * errs[0, 0]


# ------------------------------------------------------------------ algebra

def test_linear_fwd_brute_force():
    rng = np.random.default_rng(11)
    X = rng.standard_normal((3, 5))
    W = rng.standard_normal((4, 5))
    Y = o.linear_fwd(W, X)
    for t in range(3):
        for n in range(4):
            assert abs(Y[t, n] - sum(X[t, k] * W[n, k] for k in range(5))) < 1e-12


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    for i in np.ndindex(x.shape):
        x0 = x[i]
        x[i] = x0 + eps
        fp = f()
        x[i] = x0 - eps
        fm = f()
        x[i] = x0
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_linear_bwd_finite_differences():
    rng = np.random.default_rng(12)
    X, W, dY = rng.standard_normal((3, 5)), rng.standard_normal((4, 5)), rng.standard_normal((3, 4))
    L = lambda: float(np.sum(dY * o.linear_fwd(W, X)))
    dX, dW = o.linear_bwd(W, X, dY)
    assert np.allclose(dX, _fd(L, X), atol=1e-6)
    assert np.allclose(dW, _fd(L, W), atol=1e-6)


def test_mlp_relu2_and_bwd_finite_differences():
    """relu^2 is x*x for x>0 and 0 otherwise; the backward matches central
    differences of L = sum(dY * MLP(X)) for X, Wfc and Wproj."""
    rng = np.random.default_rng(13)
    X, Wfc, Wproj = rng.standard_normal((3, 4)), rng.standard_normal((8, 4)), rng.standard_normal((4, 8))
    dY = rng.standard_normal((3, 4))
    pre, h, Y = o.mlp_fwd(Wfc, Wproj, X)
    assert np.array_equal(h, np.where(pre > 0, pre * pre, 0.0))
    assert np.abs(pre).min() > 1e-3  # keep finite differences off the kink
    L = lambda: float(np.sum(dY * o.mlp_fwd(Wfc, Wproj, X)[2]))
    dX, dWfc, dWproj = o.mlp_bwd(Wfc, Wproj, X, pre, h, dY)
    assert np.allclose(dX, _fd(L, X), atol=1e-5)
    assert np.allclose(dWfc, _fd(L, Wfc), atol=1e-5)
    assert np.allclose(dWproj, _fd(L, Wproj), atol=1e-5)


def test_mlp_leaky2_and_bwd_finite_differences():
    """LeakyReLU(0.5)^2 (P1 negative result #9) is x*x for x>0 and x*x/4
    otherwise; its backward matches central differences."""
    rng = np.random.default_rng(15)
    X, Wfc, Wproj = rng.standard_normal((3, 4)), rng.standard_normal((8, 4)), rng.standard_normal((4, 8))
    dY = rng.standard_normal((3, 4))
    pre, h, Y = o.mlp_fwd(Wfc, Wproj, X, act="leaky2")
    assert np.array_equal(h, np.where(pre > 0, pre * pre, 0.25 * pre * pre))
    assert (pre < 0).any() and (pre > 0).any() and np.abs(pre).min() > 1e-3
    L = lambda: float(np.sum(dY * o.mlp_fwd(Wfc, Wproj, X, act="leaky2")[2]))
    dX, dWfc, dWproj = o.mlp_bwd(Wfc, Wproj, X, pre, h, dY, act="leaky2")
    assert np.allclose(dX, _fd(L, X), atol=1e-5)
    assert np.allclose(dWfc, _fd(L, Wfc), atol=1e-5)
    assert np.allclose(dWproj, _fd(L, Wproj), atol=1e-5)


def test_head_mlp_step_finite_differences():
    rng = np.random.default_rng(14)
    T, V, d, H = 2, 6, 4, 8
    qs = {k: {"operand": rng.standard_normal(s)} for k, s in
          (("emb", (V, d)), ("fc", (H, d)), ("proj", (d, H)))}
    X, dL = rng.standard_normal((T, d)), rng.standard_normal((T, V))
    out = o.head_mlp_step(qs["emb"], qs["fc"], qs["proj"], X, dL)
    assert np.abs(out["pre"]).min() > 1e-3
    L = lambda: float(np.sum(dL * o.head_mlp_step(qs["emb"], qs["fc"], qs["proj"], X, dL)["logits"]))
    assert np.allclose(out["dX"], _fd(L, X), atol=1e-5)
    assert np.allclose(out["dWemb"], _fd(L, qs["emb"]["operand"]), atol=1e-5)
    assert np.allclose(out["dWfc"], _fd(L, qs["fc"]["operand"]), atol=1e-5)
    assert np.allclose(out["dWproj"], _fd(L, qs["proj"]["operand"]), atol=1e-5)


def test_dw_accumulates_over_recurrence():
    """P1 "税 1": a shared weight used R times gets the sum of the R gradients;
    dW over the R token batches stacked equals the sum of per-application dW."""
    rng = np.random.default_rng(15)
    W = rng.standard_normal((4, 5))
    Xs = [rng.standard_normal((3, 5)) for _ in range(3)]
    dYs = [rng.standard_normal((3, 4)) for _ in range(3)]
    tot = sum(o.linear_bwd(W, x, g)[1] for x, g in zip(Xs, dYs))
    _, stacked = o.linear_bwd(W, np.vstack(Xs), np.vstack(dYs))
    assert np.allclose(tot, stacked, atol=1e-12)


def test_recurrent_core_is_r_applications():
    """R applications equal R single applications chained (the loop reuses the
    same quantized weights; the state is bf16 between applications)."""
    c = sy.recurrent_core_case(d=64, H=192, T=16)
    q = {"qkv": o.quantize_weight(np.concatenate([c["Wq"], c["Wk"], c["Wv"]]), 6),
         "o": o.quantize_weight(c["Wo"], 6), "fc": o.quantize_weight(c["Wfc"], 6),
         "proj": o.quantize_weight(c["Wproj"], 6)}
    X = c["X"].float().numpy()
    x3 = o.recurrent_core_fwd(q["qkv"], q["o"], q["fc"], q["proj"], X, 3, 64)
    x = X
    for _ in range(3):
        x = o.recurrent_core_fwd(q["qkv"], q["o"], q["fc"], q["proj"], x, 1, 64)
    assert np.array_equal(x3, x)
    # one application by hand from the definitions, bf16 rounding (torch's)
    # of each activation handed between GEMMs
    b = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()
    x = b(X)
    qkv = b(x @ q["qkv"]["operand"].T)
    x1 = b(x + qkv[:, :64] @ q["o"]["operand"].T)
    h = b(np.maximum(x1 @ q["fc"]["operand"].T, 0) ** 2)
    ref = b(x1 + h @ q["proj"]["operand"].T)
    one = o.recurrent_core_fwd(q["qkv"], q["o"], q["fc"], q["proj"], X, 1, 64)
    assert np.array_equal(one, ref)


def _tiny_core(rng, d, H, scale):
    nqkv = 2 * d
    ops = tuple({"operand": rng.standard_normal(shp) * scale}
                for shp in ((nqkv, d), (d, d), (H, d), (d, H)))
    return ops


@pytest.mark.parametrize("act", ["relu2", "leaky2"])
def test_recurrent_core_bwd_finite_differences(act):
    """The core's backward through R = 3 applications (exact composition, no
    bf16 rounding) matches central differences of L = sum(dY * x_R) for the
    input and for all four shared weights -- each weight's gradient is the
    sum over the three uses (P1 "税 1")."""
    rng = np.random.default_rng(21)
    d, H, T, R = 8, 24, 3, 3
    ops = _tiny_core(rng, d, H, 0.35)
    X, dY = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    out = o.recurrent_core_bwd(*ops, X, dY, R, d, act=act, exact=True)
    assert min(np.abs(s["pre"]).min() for s in out["saved"]) > 1e-3  # off the kink
    L = lambda: float(np.sum(dY * o.recurrent_core_fwd(*ops, X, R, d, act=act, exact=True)))
    assert np.allclose(out["dX"], _fd(L, X), atol=1e-5, rtol=1e-6)
    for name, k in (("dWqkv", 0), ("dWo", 1), ("dWfc", 2), ("dWproj", 3)):
        assert np.allclose(out[name], _fd(L, ops[k]["operand"]), atol=1e-5, rtol=1e-6), name
    # k and v do not reach the output when attention is left out
    assert np.all(out["dWqkv"][d:] == 0)


def test_recurrent_core_bwd_against_torch_autograd():
    """The same composition written with torch ops in float64 and
    differentiated by torch.autograd, at the small core shape d = 64."""
    rng = np.random.default_rng(22)
    d, H, T, R = 64, 192, 16, 3
    ops = _tiny_core(rng, d, H, 0.05)
    X, dY = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    out = o.recurrent_core_bwd(*ops, X, dY, R, d, exact=True)
    W = [torch.tensor(op["operand"], requires_grad=True) for op in ops]
    x = torch.tensor(X, requires_grad=True)
    s = x
    for _ in range(R):
        q = (s @ W[0].T)[:, :d]
        x1 = s + q @ W[1].T
        s = x1 + torch.relu(x1 @ W[2].T) ** 2 @ W[3].T
    (s * torch.tensor(dY)).sum().backward()
    assert np.allclose(out["out"], s.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(out["dX"], x.grad.numpy(), rtol=1e-10, atol=1e-12)
    for name, w in zip(("dWqkv", "dWo", "dWfc", "dWproj"), W):
        assert np.allclose(out[name], w.grad.numpy(), rtol=1e-10, atol=1e-12), name


def test_recurrent_core_bwd_bf16_application_by_hand():
    """One application's backward with the bf16 rounding of each materialised
    gradient (dpre, dx1, dq, dx) done by torch; the summed weight gradient over
    R = 3 equals the sum of the per-application gradients at the saved states."""
    c = sy.recurrent_core_case(d=64, H=192, T=16)
    ops = tuple(o.quantize_weight(w, 6) for w in
                (np.concatenate([c["Wq"], c["Wk"], c["Wv"]]), c["Wo"], c["Wfc"], c["Wproj"]))
    X = c["X"].float().numpy()
    dY = sy.act_bf16(np.random.default_rng(5), 16, 64, std=0.01).float().numpy()
    out = o.recurrent_core_bwd(*ops, X, dY, 3, 64)
    b = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()
    s, g = out["saved"][2], out["grads"][2]
    assert np.array_equal(g, b(dY))
    Wqkv, Wo, Wfc, Wproj = (op["operand"] for op in ops)
    dpre = b((g @ Wproj) * 2.0 * np.maximum(s["pre"], 0.0))
    dx1 = b(g + dpre @ Wfc)
    dq = b(dx1 @ Wo)
    dx = b(dx1 + dq @ Wqkv[:64])
    assert np.array_equal(out["grads"][1], dx)
    tot = {"qkv": 0.0, "o": 0.0, "fc": 0.0, "proj": 0.0}
    for r in range(3):
        s, g = out["saved"][r], out["grads"][r]
        dpre = b((g @ Wproj) * 2.0 * np.maximum(s["pre"], 0.0))
        dx1 = b(g + dpre @ Wfc)
        dq = b(dx1 @ Wo)
        tot["proj"] = tot["proj"] + g.T @ s["h"]
        tot["fc"] = tot["fc"] + dpre.T @ s["x1"]
        tot["o"] = tot["o"] + dx1.T @ s["qkv"][:, :64]
        tot["qkv"] = tot["qkv"] + np.vstack([dq.T @ s["x"], np.zeros((64, 64))])
    for k in tot:
        assert np.allclose(out["dW" + k], tot[k], rtol=1e-12, atol=1e-15), k
    for k in ("dX",):
        assert np.array_equal(out[k], b(out[k]))


# ------------------------------------------------------------- Noisy QAT

def test_philox_known_answers():
    """Philox-4x32-10 against the known-answer vectors published with the
    generator (Salmon et al., SC'11, Random123 distribution)."""
    kat = [([0, 0, 0, 0], [0, 0], [0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8]),
           ([0xffffffff] * 4, [0xffffffff] * 2, [0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd]),
           ([0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344], [0xa4093822, 0x299f31d0],
            [0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1])]
    for ctr, key, want in kat:
        assert o.philox4x32_10(ctr, key).tolist() == want


def test_noisy_weight_bounds_statistics_and_determinism():
    """P1 "幸存发现 1 Noisy QAT": the noise is (u - 0.5) * s with s the per-row
    int8 step amax/127, so |w' - w| <= s/2 (+ the fp32 rounding of the add);
    u is uniform (mean 1/2, variance 1/12, Kolmogorov-Smirnov against U(0,1));
    the same (seed, offset) gives the same weights, another offset others."""
    from scipy import stats
    W = sy.linear_case(N=512, K=512, seed=4)["W"]
    r = o.noisy_weight(W, seed=1234, offset=7)
    s = r["scales"].astype(np.float64)
    assert np.array_equal(r["scales"], o.qat_scales(W))
    d = (r["noisy"].astype(np.float64) - W.astype(np.float64)) / s[:, None]
    ulp = np.spacing(np.abs(r["noisy"])).astype(np.float64) / s[:, None]
    assert np.all(np.abs(d) <= 0.5 + ulp)
    u = (d + 0.5).ravel()
    assert abs(u.mean() - 0.5) < 0.005 and abs(u.var() - 1.0 / 12) < 0.002
    assert stats.kstest(np.clip(u, 0, 1), "uniform").pvalue > 1e-3
    assert np.array_equal(o.noisy_weight(W, 1234, 7)["noisy"], r["noisy"])
    assert not np.array_equal(o.noisy_weight(W, 1234, 8)["noisy"], r["noisy"])
    ref = torch.from_numpy(r["noisy"]).to(torch.bfloat16).float().numpy()
    assert np.array_equal(r["operand"].astype(np.float32), ref)


def test_noisy_uses_documented_counter_layout():
    """Element e takes word e % 4 of the Philox block at counter (e // 4, offset)."""
    W = np.zeros((2, 8), np.float32)
    W[:, 0] = 127.0  # s = 1 in both rows
    r = o.noisy_weight(W, seed=(5 << 32) | 9, offset=(3 << 32) | 11)
    for e in (1, 2, 5, 9, 14):
        g = e // 4
        x = o.philox4x32_10([g, 0, 11, 3], [9, 5])[e % 4]
        u = np.float32(x >> 8) * np.float32(2.0 ** -24)
        assert r["noisy"].ravel()[e] == np.float32(u - np.float32(0.5))


def test_noisy_int5_step_shares_the_draws():
    """bits = 5 scales the same uniform draws by the int5 step amax/15: a row
    of amax 15 (s = 1) gets noise u - 1/2 from the documented counter layout,
    and every |w' - w| <= s5/2."""
    W = np.zeros((2, 8), np.float32)
    W[:, 0] = 15.0
    r = o.noisy_weight(W, seed=(5 << 32) | 9, offset=(3 << 32) | 11, bits=5)
    assert np.all(r["scales"] == 1.0)
    for e in (1, 2, 5, 9, 14):
        x = o.philox4x32_10([e // 4, 0, 11, 3], [9, 5])[e % 4]
        u = np.float32(x >> 8) * np.float32(2.0 ** -24)
        assert r["noisy"].ravel()[e] == np.float32(u - np.float32(0.5))
    W = sy.linear_case(N=64, K=256, seed=6)["W"]
    r = o.noisy_weight(W, 77, 1, bits=5)
    s = r["scales"].astype(np.float64)
    assert np.array_equal(r["scales"], o.qat_scales(W, 5))
    d = np.abs(r["noisy"].astype(np.float64) - W.astype(np.float64)) / s[:, None]
    assert np.all(d <= 0.5 + np.spacing(np.abs(r["noisy"])).astype(np.float64) / s[:, None])


def test_noisy_recurrent_core_draws_per_application():
    """Application r of the noisy core uses offsets offset + 4r + (0..3); two
    applications equal one application of each draw chained."""
    c = sy.recurrent_core_case(d=64, H=192, T=8)
    Ws = [np.concatenate([c["Wq"], c["Wk"], c["Wv"]]), c["Wo"], c["Wfc"], c["Wproj"]]
    X = c["X"].float().numpy()
    two = o.recurrent_core_fwd_noisy(Ws, X, 2, 64, 3, 10)
    x = X
    for r in range(2):
        q = [{"operand": o.noisy_weight(w, 3, 10 + 4 * r + k)["operand"]} for k, w in enumerate(Ws)]
        x = o.recurrent_core_fwd(q[0], q[1], q[2], q[3], x, 1, 64)
    assert np.array_equal(two, x)
