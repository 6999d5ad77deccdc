"""GPU parity of the quantizer kernels (int5, int6, int8 grids) against the CPU
oracle: bit-exact codes,
fp32 scales, bf16 operands, fp16 export scales, fp16 passthrough and the
dequantized weights."""
import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import export as qexport
from quantization_aware_tiny_b200 import qat
from quantization_aware_tiny_b200 import synthetic as sy
from parity import bits16

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _weights():
    sd = sy.state_dict_case(n_layers=1)
    rng = np.random.default_rng(5)
    cases = {
        "cfg1_512x512_outliers": sy.linear_case()["W"],
        "fc_1536x512_heavy": sd["blocks.0.mlp.fc.weight"],
        "proj_512x1536_heavy": sd["blocks.0.mlp.proj.weight"],
        "ragged_200x136": (rng.standard_normal((200, 136)) * 0.02).astype(np.float32),
        "longrow_64x4104": (rng.standard_normal((64, 4104)) * 0.02).astype(np.float32),
        "head_8192x512": sy.head_mlp_case(T=8)["Wemb"],
    }
    z = np.zeros((8, 64), np.float32)
    z[1, 3] = 1e-30
    z[2] = 0.5
    z[3, ::2] = -7.0
    cases["degenerate_8x64"] = z
    # long staged rows: ragged widths (1040), the longest staged row (2048), a
    # width that is not a multiple of 16 (1032), and 1536-column rows whose
    # top two |w| tie or sit in different thirds of the row (a lane reduces
    # each third separately before merging) or on either side of a third
    cases["split_37x1040"] = (rng.standard_normal((37, 1040)) * 0.02).astype(np.float32)
    cases["split_9x2048"] = (rng.standard_normal((9, 2048)) * 0.02).astype(np.float32)
    cases["whole_11x1032"] = (rng.standard_normal((11, 1032)) * 0.02).astype(np.float32)
    t = (rng.standard_normal((9, 1536)) * 0.02).astype(np.float32)
    t[0, 100], t[0, 1200] = 0.5, -0.5  # max once in two thirds
    t[1, 10], t[1, 20] = 0.5, 0.5      # max twice in the first third
    t[2, 800], t[2, 1500] = 0.5, 0.25  # top two in the last two thirds
    t[3, 511], t[3, 512] = -0.4, 0.3   # top two on either side of a third
    t[4] = 0.125                       # a constant row
    t[5, 4], t[5, 516] = 0.5, -0.5     # max twice in one lane, in two thirds
    t[6, 8], t[6, 9] = 0.5, 0.5        # max twice in one group of four
    t[7, 1028], t[7, 1029] = 0.5, 0.375  # top two in one group of four
    t[8, 0], t[8, 128], t[8, 1024] = 0.25, 0.5, 0.5  # one lane holds all three
    cases["ties_9x1536"] = t
    # 512-column rows (exported three to a unit): ties and top two inside one
    # group of four, in one lane's groups, a zero row, a constant row
    t = (rng.standard_normal((7, 512)) * 0.02).astype(np.float32)
    t[0, 4], t[0, 5] = 0.5, -0.5
    t[1, 1], t[1, 129] = -0.5, 0.5
    t[2, 200], t[2, 203] = 0.5, 0.4375
    t[3] = -0.0625
    t[4] = 0.0
    t[5, 511], t[5, 0] = 0.5, 0.25
    t[6, 3], t[6, 131], t[6, 259] = 0.5, 0.5, 0.5
    cases["ties_7x512"] = t
    return cases


@pytest.mark.parametrize("bits", [5, 6, 8])
def test_quantize_weights_bit_exact(bits):
    for name, W in _weights().items():
        q = qat.quantize_weight(_dev(W), bits, keep_codes=True)
        torch.cuda.synchronize()
        ref = o.quantize_weight(W, bits)
        assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), name
        assert np.array_equal(q.scales.cpu().numpy().view(np.uint32), ref["scales"].view(np.uint32)), name
        assert np.array_equal(bits16(q.operand), o.operand_bf16_bits(ref["codes"], ref["scales"])), name
    assert qat.device_error() == 0


@pytest.mark.parametrize("bits", [5, 6, 8])
def test_export_rows_bit_exact(bits):
    rng = np.random.default_rng(9)
    ties = np.tile(np.float32([0.01, -0.03, 0.03, 0.002]), (16, 16))  # top two tie
    for name, W in list(_weights().items()) + [("ties_16x64", ties)]:
        Wd = _dev(W)
        codes = torch.empty(W.shape, dtype=torch.int8, device="cuda")
        s16 = torch.empty(W.shape[0], dtype=torch.float16, device="cuda")
        qat.quantize_rows_export(Wd, bits, codes, s16)
        torch.cuda.synchronize()
        c_ref, s_ref, _ = o.export_rows(W, bits)
        assert np.array_equal(codes.cpu().numpy(), c_ref), name
        assert np.array_equal(bits16(s16), s_ref), name


def test_export_state_dict_one_launch_bit_exact():
    """The whole 11-layer d=512 state dict (66 matrices, tied embedding, small
    tensors) in one grouped launch, against the oracle's tensor-by-tensor export."""
    sd = sy.state_dict_case()
    dev = {k: _dev(v) for k, v in sd.items()}
    n0 = qat.launch_count()
    out = qexport.export_state_dict(dev)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    ref = o.export_state_dict(sd)
    for k, r in ref.items():
        g = out[k]
        assert g["kind"] == r["kind"], k
        if r["kind"] == "fp16":
            assert np.array_equal(bits16(g["values"]).reshape(-1), r["bits16"].reshape(-1)), k
        else:
            assert np.array_equal(g["codes"].cpu().numpy(), r["codes"]), k
            assert np.array_equal(bits16(g["scale16"]), r["scale16"]), k


@pytest.mark.parametrize("flags", [{"mlp_int5": True}, {"mlp_int5": True, "attn_int5": True}])
def test_export_state_dict_mixed_int5_bit_exact(flags):
    """Mixed int5 / int6 export (MLP_INT5, ATTN_INT5) of a 3-layer state dict in
    one launch, against the oracle."""
    sd = sy.state_dict_case(n_layers=3, seed=2)
    out = qexport.export_state_dict({k: _dev(v) for k, v in sd.items()}, **flags)
    torch.cuda.synchronize()
    ref = o.export_state_dict(sd, **flags)
    assert "int5" in {r["kind"] for r in ref.values()}
    for k, r in ref.items():
        g = out[k]
        assert g["kind"] == r["kind"], k
        if r["kind"] == "fp16":
            assert np.array_equal(bits16(g["values"]).reshape(-1), r["bits16"].reshape(-1)), k
        else:
            assert np.array_equal(g["codes"].cpu().numpy(), r["codes"]), k
            assert np.array_equal(bits16(g["scale16"]), r["scale16"]), k


@pytest.mark.parametrize("bits", [5, 6])
def test_export_pack6_bit_exact(bits):
    """6-bit packed export codes (word stores for aligned full chunks, 16-bit
    stores for odd-offset rows and ragged tails, rows read from global memory
    beyond the staging buffer) equal the oracle's bit-serial packing of its
    codes; unpack_codes6 returns the oracle's codes."""
    for name, W in _weights().items():
        rows, cols = W.shape
        packed = torch.full((rows, cols * 3 // 4), 0xA5, dtype=torch.uint8, device="cuda")
        s16 = torch.empty(rows, dtype=torch.float16, device="cuda")
        Wd = _dev(W)
        qat.quantize_export_batch([(Wd, bits, packed, s16, qat.QAT_EXPORT_PACK6)])
        codes = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
        qat.unpack_codes6(packed, rows * cols, bits, codes)
        torch.cuda.synchronize()
        c_ref, s_ref, _ = o.export_rows(W, bits)
        assert np.array_equal(packed.cpu().numpy().reshape(-1), o.pack6(c_ref, bits)), name
        assert np.array_equal(bits16(s16), s_ref), name
        assert np.array_equal(codes.cpu().numpy(), c_ref), name


def test_export_state_dict_pack6_one_launch():
    """The all-int5 / int6 mixed state dict exported packed in one launch:
    packed bytes equal the oracle's packing of its codes; int8 tensors are
    unpacked codes as before."""
    sd = sy.state_dict_case(n_layers=2, seed=4)
    sd["blocks.0.attn.c_q.weight"] = sd["blocks.0.attn.c_q.weight"][:, :136].copy()  # odd row bytes
    n0 = qat.launch_count()
    out = qexport.export_state_dict({k: _dev(v) for k, v in sd.items()}, mlp_int5=True,
                                    int6_range=(0, 0), pack6=True)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    ref = o.export_state_dict(sd, mlp_int5=True, int6_start=0, int6_end=0)
    kinds = set()
    for k, r in ref.items():
        g = out[k]
        kinds.add(r["kind"])
        assert g["kind"] == r["kind"], k
        if r["kind"] in ("int5", "int6"):
            assert np.array_equal(g["packed"].cpu().numpy().reshape(-1),
                                  o.pack6(r["codes"], int(r["kind"][3:]))), k
            assert np.array_equal(bits16(g["scale16"]), r["scale16"]), k
        elif r["kind"] == "int8":
            assert np.array_equal(g["codes"].cpu().numpy(), r["codes"]), k
    assert {"int5", "int6", "int8", "fp16"} <= kinds


def _search_check(W, bits, codes, s16, rows_ok=1.0):
    """Rows whose kept candidate matches the oracle's are bit-exact; a row may
    keep another candidate only where the two candidates' errors tie to fp32
    summation accuracy (1e-5 relative), and then holds exactly that
    candidate's export."""
    c_ref, s_ref, _, ch, errs = o.export_rows_search(W, bits)
    same = (codes == c_ref).all(axis=1) & (s16 == s_ref)
    for i in np.nonzero(~same)[0]:
        alt = [k for k, q in enumerate(o.CLIP_CANDIDATES)
               if (lambda r: np.array_equal(r[0][0], codes[i]) and r[1][0] == s16[i])(
                   o.export_rows(W[i:i + 1], bits, q=q))]
        assert alt, "row %d: not the export of any candidate" % i
        assert min(abs(errs[i, k] - errs[i, ch[i]]) for k in alt) <= 1e-5 * errs[i, ch[i]], i
    assert same.mean() >= rows_ok
    return ch


@pytest.mark.parametrize("bits", [5, 6, 8])
def test_export_clip_search(bits):
    """Clip search on heavy-tailed rows of 512 and 1536 columns, a ragged
    136-column matrix and degenerate rows: bit-exact against the oracle's
    search (see _search_check for near-ties)."""
    sd = sy.state_dict_case(n_layers=1, seed=3)
    rng = np.random.default_rng(12)
    cases = [sd["blocks.0.mlp.fc.weight"], sd["blocks.0.mlp.proj.weight"],
             (rng.standard_normal((200, 136)) * 0.02).astype(np.float32), _weights()["degenerate_8x64"]]
    chosen = []
    for W in cases:
        rows, cols = W.shape
        codes = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
        s16 = torch.empty(rows, dtype=torch.float16, device="cuda")
        qat.quantize_export_batch([(_dev(W), bits, codes, s16, qat.QAT_EXPORT_CLIP_SEARCH)])
        torch.cuda.synchronize()
        chosen.append(_search_check(W, bits, codes.cpu().numpy(), bits16(s16), rows_ok=0.99))
    assert len(np.unique(np.concatenate(chosen))) >= 4   # the search is not a no-op
    assert qat.device_error() == 0


def test_export_state_dict_clip_search_packed():
    """A whole state dict with clip search and 6-bit packing in one launch."""
    sd = sy.state_dict_case(n_layers=2, seed=6)
    out = qexport.export_state_dict({k: _dev(v) for k, v in sd.items()}, pack6=True,
                                    clip_search=True)
    torch.cuda.synchronize()
    for k, r in o.export_state_dict(sd).items():
        g = out[k]
        if r["kind"] == "int6":
            codes = o.unpack6(g["packed"].cpu().numpy(), sd[k].size, 6).reshape(sd[k].shape)
            _search_check(sd[k], 6, codes, bits16(g["scale16"]), rows_ok=0.99)
        elif r["kind"] == "int8":
            _search_check(sd[k], 8, g["codes"].cpu().numpy(), bits16(g["scale16"]), rows_ok=0.99)


def test_dequantize_rows_bit_exact():
    sd = sy.state_dict_case(n_layers=1)
    for name in ("blocks.0.mlp.fc.weight", "blocks.0.attn.c_k.weight"):
        W = sd[name]
        c, s16, _ = o.export_rows(W, 6)
        cd, sd16 = _dev(c), _dev(s16.view(np.float16))
        out32 = torch.empty(W.shape, dtype=torch.float32, device="cuda")
        out16 = torch.empty(W.shape, dtype=torch.bfloat16, device="cuda")
        qat.dequantize_rows(cd, sd16, out32)
        qat.dequantize_rows(cd, sd16, out16)
        torch.cuda.synchronize()
        ref = o.dequant_export(c, s16)
        assert np.array_equal(out32.cpu().numpy().view(np.uint32), ref.view(np.uint32)), name
        assert np.array_equal(bits16(out16), o.bf16_bits(ref)), name


def test_dequantize_rows_batch_one_launch():
    """The roundtrip of a whole exported state dict (3 layers: 18 int6 tensors
    of 256-1536 columns, plus a ragged 200 x 136 int8 tensor) in one grouped
    launch, fp32 and bf16 outputs mixed: bit-exact with the oracle."""
    sd = sy.state_dict_case(n_layers=3, seed=6)
    rng = np.random.default_rng(6)
    W = {k: v for k, v in sd.items() if v.ndim == 2 and v.size > 65536 and "tok_emb" not in k}
    W["ragged"] = (rng.standard_normal((200, 136)) * 0.02).astype(np.float32)
    items, refs = [], []
    for i, (name, w) in enumerate(sorted(W.items())):
        c, s16, _ = o.export_rows(w, 8 if name == "ragged" else 6)
        out = torch.full(w.shape, float("nan"), device="cuda",
                         dtype=torch.bfloat16 if i % 2 else torch.float32)
        items.append((_dev(c), _dev(s16.view(np.float16)), out))
        refs.append((name, o.dequant_export(c, s16)))
    n0 = qat.launch_count()
    qat.dequantize_rows_batch(items)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    for (name, ref), (_, _, out) in zip(refs, items):
        if out.dtype == torch.float32:
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32)), name
        else:
            assert np.array_equal(bits16(out), o.bf16_bits(ref)), name


def test_export_and_dequantize_past_96_descriptors():
    """More descriptors than the mid-size parameter block holds (100 small
    weights of assorted shapes, int6 / int8 / int5, and two fp16 passthrough
    tensors): one export launch and one grouped dequantize launch, both
    bit-exact with the oracle."""
    rng = np.random.default_rng(31)
    shapes = [(8 + 8 * (i % 5), (16, 64, 136, 512)[i % 4]) for i in range(100)]
    bits = [(6, 8, 5)[i % 3] for i in range(100)]
    Ws = [(rng.standard_normal(sh) * 0.02).astype(np.float32) for sh in shapes]
    descs, outs = [], []
    for w, b in zip(Ws, bits):
        codes = torch.empty(w.shape, dtype=torch.int8, device="cuda")
        s16 = torch.empty(w.shape[0], dtype=torch.float16, device="cuda")
        descs.append((_dev(w), b, codes, s16))
        outs.append((codes, s16))
    flat = [(rng.standard_normal(300) * 0.02).astype(np.float32) for _ in range(2)]
    f16 = [torch.empty(300, dtype=torch.float16, device="cuda") for _ in flat]
    for f, o16 in zip(flat, f16):
        descs.append((_dev(f), qat.QAT_EXPORT_FP16, o16, None))
    n0 = qat.launch_count()
    qat.quantize_export_batch(descs)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    items, refs = [], []
    for i, (w, b, (codes, s16)) in enumerate(zip(Ws, bits, outs)):
        c_ref, s_ref, _ = o.export_rows(w, b)
        assert np.array_equal(codes.cpu().numpy(), c_ref), i
        assert np.array_equal(bits16(s16), s_ref), i
        out = torch.full(w.shape, float("nan"), device="cuda",
                         dtype=torch.bfloat16 if i % 2 else torch.float32)
        items.append((codes, s16, out))
        refs.append(o.dequant_export(c_ref, s_ref))
    for f, o16 in zip(flat, f16):
        assert np.array_equal(bits16(o16), f.astype(np.float16).view(np.uint16))
    n0 = qat.launch_count()
    qat.dequantize_rows_batch(items)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    for i, (ref, (_, _, out)) in enumerate(zip(refs, items)):
        if out.dtype == torch.float32:
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32)), i
        else:
            assert np.array_equal(bits16(out), o.bf16_bits(ref)), i
    assert qat.device_error() == 0


def _near_tie_rows(n_rows=256, cols=512, seed=21, levels=127):
    """Rows whose entries sit within a few ulps of (k + 1/2) * s: the code then
    depends on the correctly rounded quotient w / s (and on ties going to
    even).  The first two entries carry the row's |w| maximum, so both the
    training scale and the export clip equal amax / levels."""
    rng = np.random.default_rng(seed)
    W = np.empty((n_rows, cols), np.float32)
    for i in range(n_rows):
        amax = np.float32(rng.uniform(1e-3, 1e2))
        s = amax / np.float32(levels)
        k = rng.integers(-levels, levels, cols).astype(np.float32)
        base = (k + np.float32(0.5)) * s
        steps = rng.integers(-3, 4, cols)
        w = base.copy()
        for st in range(1, 4):
            w = np.where(steps >= st, np.nextafter(w, np.float32(np.inf)), w)
            w = np.where(steps <= -st, np.nextafter(w, np.float32(-np.inf)), w)
        w = np.clip(w, -amax, amax)
        w[0], w[1] = amax, -amax
        W[i] = w
    return W


@pytest.mark.parametrize("bits", [5, 6, 8])
def test_near_tie_quotients_bit_exact(bits):
    """Pins the division w / s and the two roundings against the oracle's
    IEEE fp32 division on adversarial near-tie inputs, for both the training
    quantizer and the export quantizer."""
    W = _near_tie_rows(levels=15 if bits == 5 else 127)
    q = qat.quantize_weight(_dev(W), bits, keep_codes=True)
    codes = torch.empty(W.shape, dtype=torch.int8, device="cuda")
    s16 = torch.empty(W.shape[0], dtype=torch.float16, device="cuda")
    qat.quantize_rows_export(_dev(W), bits, codes, s16)
    torch.cuda.synchronize()
    ref = o.quantize_weight(W, bits)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    c_ref, s_ref, _ = o.export_rows(W, bits)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(bits16(s16), s_ref)


def test_quantize_weights_batch_one_launch():
    """Several weights (mixed grids and widths) quantized in one launch equal
    the oracle bit for bit, as one call per weight does."""
    ws = _weights()
    names = ["head_8192x512", "fc_1536x512_heavy", "proj_512x1536_heavy", "ragged_200x136",
             "longrow_64x4104", "degenerate_8x64"]
    bits = [8, 6, 6, 5, 6, 8]
    Ws = [_dev(ws[n]) for n in names]
    n0 = qat.launch_count()
    qs = qat.quantize_weights(Ws, bits, keep_codes=True)
    torch.cuda.synchronize()
    assert qat.launch_count() - n0 == 1
    for n, b, q in zip(names, bits, qs):
        ref = o.quantize_weight(ws[n], b)
        assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), n
        assert np.array_equal(q.scales.cpu().numpy().view(np.uint32), ref["scales"].view(np.uint32)), n
        assert np.array_equal(bits16(q.operand), o.operand_bf16_bits(ref["codes"], ref["scales"])), n
    assert qat.device_error() == 0
