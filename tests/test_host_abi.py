"""Host-side checks that need no GPU: the C-ABI library loads and exports every
symbol include/qat.h declares, argument validation rejects bad calls before
any launch, and the export planner applies the passthrough rules."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as o
from quantization_aware_tiny_b200 import build, qat
from quantization_aware_tiny_b200 import export as qexport
from quantization_aware_tiny_b200 import synthetic as sy

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qat.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return qat.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|int64_t|size_t|char\s*\*|const char\s*\*)\s*\*?\s*(\w+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_symbols_exported(L):
    names = _declared()
    assert set(names) == set(qat.EXPORTED), names
    for n in names:
        assert hasattr(L, n), n


def test_strerror_and_workspace_sizes(L):
    assert qat.strerror(0) == "ok"
    assert "aligned" in qat.strerror(qat.QAT_ERR_ALIGN)
    assert qat.strerror(99) == "unknown error"
    # raw weights: bf16 operand + fp32 scales, each rounded up to 256 bytes
    # raw weights: the operand and scales (a NULL workspace instead selects the
    # fused quantizing producer where it applies)
    assert qat.workspace_size(qat.QAT_OP_LINEAR_FWD, 512, 512, 256, True) == 512 * 512 * 2 + 2048
    assert qat.workspace_size(qat.QAT_OP_LINEAR_BWD, 512, 512, 256, True) == 512 * 512 * 2 + 2048
    assert qat.workspace_size(qat.QAT_OP_MLP_FWD, 512, 1536, 100, True) == (
        100 * 1536 * 2 + 2 * (512 * 1536 * 2) + 2048 + 6144)
    assert qat.workspace_size(qat.QAT_OP_LINEAR_FWD, 512, 512, 256, False) == 0
    assert qat.workspace_size(qat.QAT_OP_MLP_BWD, 512, 1536, 8192, False) == 8192 * 1536 * 2
    assert qat.workspace_size(qat.QAT_OP_MLP_FWD, 0, 1536, 8192, False) == 0


P = ctypes.c_void_p


def test_argument_validation_before_launch(L):
    """Bad calls return an error code and launch nothing (no GPU is touched)."""
    before = qat.launch_count()
    A16, A_BAD = P(0x10000), P(0x10004)
    # null activations / outputs
    assert L.qat_linear_fwd(A16, None, 512, 512, 6, None, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_ARG
    # bits outside {5, 6, 8}
    assert L.qat_linear_fwd(A16, None, 512, 512, 7, A16, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_ARG
    assert L.qat_linear_fwd(A16, None, 512, 512, 4, A16, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_ARG
    # feature dims must be multiples of 8
    assert L.qat_linear_fwd(A16, None, 500, 512, 6, A16, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_SHAPE
    # both W and qw, or neither
    assert L.qat_linear_fwd(None, None, 512, 512, 6, A16, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_ARG
    # misaligned weights
    assert L.qat_quantize_weights(A_BAD, 512, 512, 6, None, A16, None, None) == qat.QAT_ERR_ALIGN
    # the wait-timeout diagnostic: limit outside 1 us .. 10 s
    assert L.qat_selftest_wait_timeout(999, None) == qat.QAT_ERR_ARG
    assert L.qat_selftest_wait_timeout(10000000001, None) == qat.QAT_ERR_ARG
    # batched quantize: descriptor count, null pointers, bits, shape, alignment
    Q = qat._QuantDesc
    ok = Q(0x10000, None, 0x10000, 0x10000, 512, 512, 6, 0)
    arr = (Q * 17)(*([ok] * 17))
    assert L.qat_quantize_weights_batch(None, 1, None) == qat.QAT_ERR_ARG
    assert L.qat_quantize_weights_batch(ctypes.cast(arr, ctypes.c_void_p), 0, None) == qat.QAT_ERR_ARG
    assert L.qat_quantize_weights_batch(ctypes.cast(arr, ctypes.c_void_p), 17, None) == qat.QAT_ERR_ARG
    for bad, rc in ((Q(0x10000, None, None, 0x10000, 512, 512, 6, 0), qat.QAT_ERR_ARG),
                    (Q(0x10000, None, 0x10000, 0x10000, 512, 512, 7, 0), qat.QAT_ERR_ARG),
                    (Q(0x10000, None, 0x10000, 0x10000, 512, 500, 6, 0), qat.QAT_ERR_SHAPE),
                    (Q(0x10004, None, 0x10000, 0x10000, 512, 512, 6, 0), qat.QAT_ERR_ALIGN)):
        two = (Q * 2)(ok, bad)  # the bad descriptor second: nothing launches for the first either
        assert L.qat_quantize_weights_batch(ctypes.cast(two, ctypes.c_void_p), 2, None) == rc
    # workspace too small for raw weights
    assert L.qat_linear_fwd(A16, None, 512, 512, 6, A16, 0, 256, None, A16, A16, 1024, None) == qat.QAT_ERR_WORKSPACE
    # no workspace and no fused path (fewer than 256 tokens, or K > 1024)
    assert L.qat_linear_fwd(A16, None, 512, 512, 6, A16, 0, 255, None, A16, None, 0, None) == qat.QAT_ERR_WORKSPACE
    assert L.qat_linear_fwd(A16, None, 512, 2048, 6, A16, 0, 4096, None, A16, None, 0, None) == qat.QAT_ERR_WORKSPACE
    # fused path: misaligned fp32 weights
    assert L.qat_linear_fwd(A_BAD, None, 512, 512, 6, A16, 0, 256, None, A16, None, 0, None) == qat.QAT_ERR_ALIGN
    # export: longer rows than the top-2 quantile covers, bad mode, too many descs
    assert L.quantize_rows_export(A16, 4, 1 << 21, 6, A16, A16, None) == qat.QAT_ERR_SHAPE
    assert L.quantize_rows_export(A16, 4, 700000, 6, A16, A16, None) == qat.QAT_ERR_SHAPE
    assert L.quantize_rows_export(A16, 4, 512, 7, A16, A16, None) == qat.QAT_ERR_ARG
    assert L.quantize_export_batch(None, 1, None) == qat.QAT_ERR_ARG
    assert L.quantize_export_batch(A16, 257, None) == qat.QAT_ERR_ARG
    assert L.dequantize_rows(A16, A16, 4, 12, 0, A16, None) == qat.QAT_ERR_SHAPE
    # 6-bit packing: only int5 / int6, unknown flags refused, n a multiple of 8
    bad = (qat._ExportDesc * 3)(qat._ExportDesc(0x10000, 4, 512, 8, qat.QAT_EXPORT_PACK6, 0x10000, 0x10000),
                                qat._ExportDesc(0x10000, 4, 512, 6, 8, 0x10000, 0x10000),
                                qat._ExportDesc(0x10000, 4, 512, qat.QAT_EXPORT_FP16, 1, 0x10000, 0))
    for i in range(3):
        assert L.quantize_export_batch(ctypes.byref(bad[i]), 1, None) == qat.QAT_ERR_ARG
    # clip search: not for fp16 passthrough, rows of at most 2048 columns, unknown flag 4
    srch = (qat._ExportDesc * 3)(
        qat._ExportDesc(0x10000, 4, 512, qat.QAT_EXPORT_FP16, qat.QAT_EXPORT_CLIP_SEARCH, 0x10000, 0),
        qat._ExportDesc(0x10000, 4, 4096, 6, qat.QAT_EXPORT_CLIP_SEARCH, 0x10000, 0x10000),
        qat._ExportDesc(0x10000, 4, 512, 6, 4, 0x10000, 0x10000))
    assert L.quantize_export_batch(ctypes.byref(srch[0]), 1, None) == qat.QAT_ERR_ARG
    assert L.quantize_export_batch(ctypes.byref(srch[1]), 1, None) == qat.QAT_ERR_SHAPE
    assert L.quantize_export_batch(ctypes.byref(srch[2]), 1, None) == qat.QAT_ERR_ARG
    assert L.unpack_codes6(A16, 12, 6, A16, None) == qat.QAT_ERR_SHAPE
    assert L.unpack_codes6(A16, 16, 8, A16, None) == qat.QAT_ERR_ARG
    assert L.unpack_codes6(A_BAD, 16, 6, A16, None) == qat.QAT_ERR_ALIGN
    assert L.dequantize_rows(A16, A16, 4, 16, 3, A16, None) == qat.QAT_ERR_ARG
    # grouped dequantize: count, null array, then a bad descriptor after a good one
    D = qat._DequantDesc
    good = D(0x10000, 0x10000, 4, 16, qat.QAT_DTYPE_F32, 0, 0x10000)
    assert L.dequantize_rows_batch(None, 1, None) == qat.QAT_ERR_ARG
    many = (D * 257)(*([good] * 257))
    assert L.dequantize_rows_batch(ctypes.cast(many, ctypes.c_void_p), 0, None) == qat.QAT_ERR_ARG
    assert L.dequantize_rows_batch(ctypes.cast(many, ctypes.c_void_p), 257, None) == qat.QAT_ERR_ARG
    for bad, rc in ((D(0x10000, None, 4, 16, 0, 0, 0x10000), qat.QAT_ERR_ARG),
                    (D(0x10000, 0x10000, 4, 16, 2, 0, 0x10000), qat.QAT_ERR_ARG),
                    (D(0x10000, 0x10000, -1, 16, 0, 0, 0x10000), qat.QAT_ERR_ARG),
                    (D(0x10000, 0x10000, 4, 12, 0, 0, 0x10000), qat.QAT_ERR_SHAPE),
                    (D(0x10000, 0x10000, 4, 16, 0, 0, 0x10008), qat.QAT_ERR_ALIGN)):
        two = (D * 2)(good, bad)
        assert L.dequantize_rows_batch(ctypes.cast(two, ctypes.c_void_p), 2, None) == rc
    # more 1,024-item tiles (one thread block each) than a grid can hold: 2^40 rows of 16
    assert L.dequantize_rows(A16, A16, 1 << 40, 16, 0, A16, None) == qat.QAT_ERR_SHAPE
    huge = (D * 2)(good, D(0x10000, 0x10000, 1 << 40, 16, 0, 0, 0x10000))
    assert L.dequantize_rows_batch(ctypes.cast(huge, ctypes.c_void_p), 2, None) == qat.QAT_ERR_SHAPE
    assert L.qat_mlp_bwd(None, None, None, None, 512, 1536, 6, 0, A16, A16, None, A16, 8, None,
                         None, None, None, None, 0, None, 0, None) == qat.QAT_ERR_ARG
    # a dX residual needs dX; the X row stride is at least K and a multiple of 8
    assert L.qat_mlp_bwd(None, None, None, None, 512, 1536, 6, 0, A16, A16, A16, A16, 8, A16,
                         None, None, None, None, 0, None, 0, None) == qat.QAT_ERR_ARG
    assert L.qat_linear_bwd(None, None, 512, 512, 6, A16, 0, A16, 8, A16, None, A16, 0, None, 0,
                            None) == qat.QAT_ERR_ARG
    assert L.qat_linear_bwd(None, None, 512, 512, 6, A16, 256, A16, 8, None, None, A16, 0, None, 0,
                            None) == qat.QAT_ERR_SHAPE
    assert L.qat_linear_bwd(None, None, 512, 512, 6, A16, 516, A16, 8, None, None, A16, 0, None, 0,
                            None) == qat.QAT_ERR_SHAPE
    # activation outside {relu^2, leaky^2}; bits 7
    assert L.qat_mlp_fwd(None, None, None, None, 512, 1536, 6, 2, A16, 8, None, A16, None, None,
                         None, 0, None) == qat.QAT_ERR_ARG
    assert L.qat_noisy_operand(A16, 4, 512, 7, 1, 0, None, A16, None) == qat.QAT_ERR_ARG
    assert qat.launch_count() == before


def test_export_plan_matches_page_rules():
    """The product planner and the oracle's own rule implementation agree on
    every tensor of the 11-layer state dict and on the boundary cases."""
    sd = sy.state_dict_case()
    sd["blocks.0.edge"] = np.zeros((256, 256), np.float32)      # exactly 65,536
    sd["blocks.12.big"] = np.ones((300, 256), np.float32)       # outside 0..10
    sd["flat"] = np.zeros(70000, np.float32)                   # not 2-D
    kinds = {n: ("fp16" if m == qat.QAT_EXPORT_FP16 else "int%d" % m)
             for n, m in qexport.plan({k: _Shape(v) for k, v in sd.items()})}
    oref = o.export_state_dict(sd)
    assert kinds == {k: v["kind"] for k, v in oref.items()}
    assert kinds["blocks.3.mlp.fc.weight"] == "int6" and kinds["blocks.12.big"] == "int8"
    assert kinds["blocks.0.edge"] == "fp16" and kinds["tok_emb.weight"] == "fp16"
    off = {n: m for n, m in qexport.plan({k: _Shape(v) for k, v in sd.items()}, int6_range=(-1, -1))}
    assert off["blocks.3.mlp.fc.weight"] == 8
    for flags in ({"mlp_int5": True}, {"attn_int5": True}, {"mlp_int5": True, "attn_int5": True}):
        k5 = {n: ("fp16" if m == qat.QAT_EXPORT_FP16 else "int%d" % m)
              for n, m in qexport.plan({k: _Shape(v) for k, v in sd.items()}, **flags)}
        assert k5 == {k: v["kind"] for k, v in o.export_state_dict(sd, **flags).items()}
        assert (k5["blocks.3.mlp.fc.weight"] == "int5") == ("mlp_int5" in flags)
        assert (k5["blocks.3.attn.c_q.weight"] == "int5") == ("attn_int5" in flags)


class _Shape:
    def __init__(self, a):
        self.shape = a.shape
        self._n = a.size

    def numel(self):
        return self._n


def test_export_quantile_parameters_cover_page_row_lengths():
    """Rows up to 625,001 columns need only the top-2 order statistics."""
    for n in (512, 1536, 2048, 625001):
        pos = 0.9999984 * (n - 1)
        assert n - int(np.floor(pos)) <= 2
    assert 700000 - int(np.floor(0.9999984 * 699999)) > 2
