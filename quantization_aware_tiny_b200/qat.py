"""Thin ctypes binding of the sm_100a C-ABI library ``libqat_b200.so``.

Argument marshalling only: every function passes tensor data pointers, sizes
and the current CUDA stream to the C entry point of the same name
(include/qat.h) and raises ``QatError`` on a non-zero status.  All compute
runs in the library's kernels.  If the library is missing, ``lib()`` raises:
there is no CPU or PyTorch fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqat_b200.so")

QAT_OK = 0
QAT_ERR_ARG, QAT_ERR_ALIGN, QAT_ERR_SHAPE, QAT_ERR_WORKSPACE = 1, 2, 3, 4
QAT_ERR_CUDA, QAT_ERR_TIMEOUT, QAT_ERR_UNSUPPORTED = 5, 6, 7
QAT_OP_LINEAR_FWD, QAT_OP_LINEAR_BWD, QAT_OP_MLP_FWD, QAT_OP_MLP_BWD = 1, 2, 3, 4
QAT_EXPORT_FP16 = 16
QAT_EXPORT_MAX_DESCS = 256
QAT_DTYPE_F32, QAT_DTYPE_BF16 = 0, 1

# every symbol include/qat.h declares
EXPORTED = ("qat_strerror", "qat_launch_count", "qat_device_error", "qat_quantize_weights",
            "qat_workspace_size", "qat_linear_fwd", "qat_linear_bwd", "qat_mlp_fwd",
            "qat_mlp_bwd", "quantize_rows_export", "quantize_export_batch", "dequantize_rows",
            "qat_linear_fwd_noalloc", "qat_noisy_operand", "unpack_codes6",
            "qat_quantize_weights_batch", "qat_selftest_wait_timeout", "dequantize_rows_batch")
QAT_EXPORT_PACK6 = 1
QAT_EXPORT_CLIP_SEARCH = 2
QAT_ACT_RELU2 = 0
QAT_ACT_LEAKY_RELU2 = 1
_ACTS = {"relu2": QAT_ACT_RELU2, "leaky2": QAT_ACT_LEAKY_RELU2}
QAT_NOALLOC_MAX_ELEMS = 4194304
QAT_NOALLOC_MAX_ROWS = 16384


class QatError(RuntimeError):
    def __init__(self, code, where):
        super().__init__("%s: %s (code %d)" % (where, strerror(code), code))
        self.code = code


class _QWeight(ctypes.Structure):
    _fields_ = [("operand", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("bits", ctypes.c_int32)]


class _QuantDesc(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("operand", ctypes.c_void_p), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("pad", ctypes.c_int32)]


class _DequantDesc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("out_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("out", ctypes.c_void_p)]


QAT_DEQUANT_MAX_DESCS = 256


class _ExportDesc(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("mode", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("dst", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libqat_b200.so (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libqat_b200.so is not built (python -m quantization_aware_tiny_b200.build);"
                              " there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.qat_strerror.argtypes = [ctypes.c_int]
        L.qat_strerror.restype = ctypes.c_char_p
        L.qat_launch_count.argtypes = []
        L.qat_launch_count.restype = I64
        L.qat_device_error.argtypes = [P]
        L.qat_quantize_weights.argtypes = [P, I32, I32, I32, P, P, P, P]
        L.qat_quantize_weights_batch.argtypes = [P, I32, P]
        L.qat_selftest_wait_timeout.argtypes = [I64, P]
        L.qat_workspace_size.argtypes = [I32, I32, I32, I64, I32]
        L.qat_workspace_size.restype = SZ
        L.qat_linear_fwd.argtypes = [P, P, I32, I32, I32, P, I64, I64, P, P, P, SZ, P]
        L.qat_linear_bwd.argtypes = [P, P, I32, I32, I32, P, I64, P, I64, P, P, P, I32, P, SZ, P]
        L.qat_mlp_fwd.argtypes = [P, P, P, P, I32, I32, I32, I32, P, I64, P, P, P, P, P, SZ, P]
        L.qat_mlp_bwd.argtypes = [P, P, P, P, I32, I32, I32, I32, P, P, P, P, I64, P, P, P, P, P,
                                  I32, P, SZ, P]
        L.quantize_rows_export.argtypes = [P, I64, I64, I32, P, P, P]
        L.quantize_export_batch.argtypes = [P, I32, P]
        L.dequantize_rows.argtypes = [P, P, I64, I64, I32, P, P]
        L.dequantize_rows_batch.argtypes = [P, I32, P]
        L.unpack_codes6.argtypes = [P, I64, I32, P, P]
        L.qat_linear_fwd_noalloc.argtypes = [P, I32, I32, I32, P, I64, I64, P, P, P]
        L.qat_noisy_operand.argtypes = [P, I32, I32, I32, ctypes.c_uint64, ctypes.c_uint64, P, P,
                                        P]
        for name in EXPORTED:
            if name not in ("qat_strerror", "qat_launch_count", "qat_workspace_size"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def strerror(code):
    return lib().qat_strerror(int(code)).decode()


def _check(rc, where):
    if rc != QAT_OK:
        raise QatError(rc, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ws(ws):
    if ws is None:
        return None, 0
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


class QWeight:
    """A quantized weight on the device (the STE operand / recurrence cache).
    Holds its tensors so the pointers handed to the library stay valid."""

    def __init__(self, operand, scales, codes, bits):
        self.operand, self.scales, self.codes, self.bits = operand, scales, codes, bits
        self.N, self.K = operand.shape

    def struct(self):
        return _QWeight(self.operand.data_ptr(),
                        self.scales.data_ptr() if self.scales is not None else None,
                        self.codes.data_ptr() if self.codes is not None else None,
                        self.N, self.K, self.bits)


def _qref(q):
    return None if q is None else ctypes.byref(q.struct())


def launch_count():
    return int(lib().qat_launch_count())


def device_error(stream=None):
    """Synchronizes the stream and returns the device error code (0 = none)."""
    return int(lib().qat_device_error(_stream(stream)))


def workspace_size(op, a, b, T, raw_weights):
    return int(lib().qat_workspace_size(op, a, b, T, int(bool(raw_weights))))


def qat_selftest_wait_timeout(limit_ns, stream=None):
    """Diagnostic: a bounded device wait that runs out after limit_ns and
    records QAT_ERR_TIMEOUT for the next device_error()."""
    _check(lib().qat_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "qat_selftest_wait_timeout")


def qat_quantize_weights(W, bits, scales, codes=None, operand=None, stream=None):
    """scales [N] fp32 (required); codes [N,K] int8 and operand [N,K] bf16 are
    written when given."""
    N, K = W.shape
    _check(lib().qat_quantize_weights(_p(W), N, K, bits, _p(codes), _p(scales), _p(operand),
                                      _stream(stream)), "qat_quantize_weights")


QAT_QUANT_MAX_DESCS = 16


def qat_quantize_weights_batch(items, stream=None):
    """items: (W, bits, scales, codes, operand) per weight (codes / operand may
    be None); one launch for all of them."""
    arr = (_QuantDesc * len(items))()
    for i, (W, bits, scales, codes, operand) in enumerate(items):
        N, K = W.shape
        arr[i] = _QuantDesc(W.data_ptr(), _p(codes), _p(scales), _p(operand), N, K, bits, 0)
    _check(lib().qat_quantize_weights_batch(ctypes.cast(arr, ctypes.c_void_p), len(items),
                                            _stream(stream)), "qat_quantize_weights_batch")


def quantize_weights(Ws, bits, keep_codes=False, stream=None):
    """Quantize several weights (bits: one per weight, or one for all) in one
    launch into new QWeights."""
    bits = list(bits) if isinstance(bits, (list, tuple)) else [bits] * len(Ws)
    out = []
    for W, b in zip(Ws, bits):
        N, K = W.shape
        out.append(QWeight(torch.empty((N, K), dtype=torch.bfloat16, device=W.device),
                           torch.empty(N, dtype=torch.float32, device=W.device),
                           torch.empty((N, K), dtype=torch.int8, device=W.device) if keep_codes else None,
                           b))
    qat_quantize_weights_batch([(W, q.bits, q.scales, q.codes, q.operand) for W, q in zip(Ws, out)],
                               stream)
    return out


def quantize_weight(W, bits, keep_codes=False, stream=None):
    """Quantize once into a new QWeight (the per-step operand or the recurrence cache)."""
    N, K = W.shape
    scales = torch.empty(N, dtype=torch.float32, device=W.device)
    operand = torch.empty((N, K), dtype=torch.bfloat16, device=W.device)
    codes = torch.empty((N, K), dtype=torch.int8, device=W.device) if keep_codes else None
    qat_quantize_weights(W, bits, scales, codes, operand, stream)
    return QWeight(operand, scales, codes, bits)


def qat_noisy_operand(W, seed, offset, operand, scales=None, stream=None, bits=8):
    """Noisy-QAT forward operand bf16(w + (u - 1/2) * amax/L) of W [N,K]; L = 127
    (the int8 step) for bits 6 / 8, 15 (the int5 step) for bits 5."""
    N, K = W.shape
    _check(lib().qat_noisy_operand(_p(W), N, K, int(bits), int(seed), int(offset), _p(scales),
                                   _p(operand), _stream(stream)), "qat_noisy_operand")


def noisy_weight(W, seed, offset, stream=None, bits=8):
    """A new QWeight holding the Noisy-QAT operand of W (bits recorded as 0)."""
    N, K = W.shape
    scales = torch.empty(N, dtype=torch.float32, device=W.device)
    operand = torch.empty((N, K), dtype=torch.bfloat16, device=W.device)
    qat_noisy_operand(W, seed, offset, operand, scales, stream, bits=bits)
    return QWeight(operand, scales, None, 0)


def qat_linear_fwd(X, Y, bits, W=None, qw=None, residual=None, workspace=None, N=None, K=None,
                   ldx=0, T=None, stream=None):
    if N is None:
        N, K = (qw.N, qw.K) if qw is not None else W.shape
    if T is None:
        T = X.shape[0]
    ws, wsb = _ws(workspace)
    _check(lib().qat_linear_fwd(_p(W), _qref(qw), N, K, bits, _p(X), ldx, T, _p(residual), _p(Y),
                                ws, wsb, _stream(stream)), "qat_linear_fwd")


def qat_linear_bwd(X, dY, bits, W=None, qw=None, dX=None, dW=None, accumulate_dW=False,
                   workspace=None, N=None, K=None, ldx=0, dX_residual=None, stream=None):
    """dX = bf16(dY . Wq (+ dX_residual)); dW (+)= dY^T . X (X rows ldx apart)."""
    if N is None:
        N, K = (qw.N, qw.K) if qw is not None else ((W.shape) if W is not None else dW.shape)
    ws, wsb = _ws(workspace)
    _check(lib().qat_linear_bwd(_p(W), _qref(qw), N, K, bits, _p(X), ldx, _p(dY), dY.shape[0],
                                _p(dX_residual), _p(dX), _p(dW), int(bool(accumulate_dW)), ws, wsb,
                                _stream(stream)), "qat_linear_bwd")


def qat_mlp_fwd(X, Y, bits, d, H, Wfc=None, Wproj=None, qfc=None, qproj=None, residual=None,
                pre_save=None, h_save=None, workspace=None, stream=None, act="relu2"):
    """act = "relu2" (relu(x)^2) or "leaky2" (leaky_relu(x, 0.5)^2)."""
    ws, wsb = _ws(workspace)
    _check(lib().qat_mlp_fwd(_p(Wfc), _p(Wproj), _qref(qfc), _qref(qproj), d, H, bits,
                             _ACTS[act], _p(X),
                             X.shape[0], _p(residual), _p(Y), _p(pre_save), _p(h_save), ws, wsb,
                             _stream(stream)), "qat_mlp_fwd")


def qat_mlp_bwd(X, pre, h, dY, bits, d, H, Wfc=None, Wproj=None, qfc=None, qproj=None, dX=None,
                dWfc=None, dWproj=None, accumulate_dW=False, workspace=None, stream=None,
                act="relu2", dX_residual=None, dpre_save=None):
    ws, wsb = _ws(workspace)
    _check(lib().qat_mlp_bwd(_p(Wfc), _p(Wproj), _qref(qfc), _qref(qproj), d, H, bits,
                             _ACTS[act], _p(X),
                             _p(pre), _p(h), _p(dY), X.shape[0], _p(dX_residual), _p(dX),
                             _p(dpre_save), _p(dWfc), _p(dWproj), int(bool(accumulate_dW)), ws,
                             wsb, _stream(stream)), "qat_mlp_bwd")


def quantize_rows_export(W, bits, codes, scales, stream=None):
    rows, cols = W.shape
    _check(lib().quantize_rows_export(_p(W), rows, cols, bits, _p(codes), _p(scales),
                                      _stream(stream)), "quantize_rows_export")


def export_descs(descs):
    """Marshal (src, mode, dst, scales[, flags]) tuples into the C descriptor
    array once; the result can be passed to quantize_export_batch repeatedly."""
    arr = (_ExportDesc * len(descs))()
    for i, dsc in enumerate(descs):
        src, mode, dst, scales = dsc[:4]
        flags = dsc[4] if len(dsc) > 4 else 0
        rows, cols = (src.shape if src.dim() == 2 else (1, src.numel()))
        arr[i] = _ExportDesc(src.data_ptr(), rows, cols, mode, flags, dst.data_ptr(),
                             scales.data_ptr() if scales is not None else None)
    return arr


def quantize_export_batch(descs, stream=None):
    """descs: list of (src, mode, dst, scales[, flags]) with src a 2-D (or flat)
    fp32 device tensor, mode 5 / 6 / 8 / QAT_EXPORT_FP16, flags 0 or an OR of
    QAT_EXPORT_PACK6 / QAT_EXPORT_CLIP_SEARCH -- or an array from export_descs()
    (the tensors it points to must stay alive)."""
    arr = descs if isinstance(descs, ctypes.Array) else export_descs(descs)
    _check(lib().quantize_export_batch(arr, len(arr), _stream(stream)), "quantize_export_batch")


def unpack_codes6(packed, n, bits, codes, stream=None):
    """n 6-bit packed codes (uint8 device tensor of 3n/4 bytes) into int8 codes."""
    _check(lib().unpack_codes6(_p(packed), int(n), int(bits), _p(codes), _stream(stream)),
           "unpack_codes6")


def dequantize_rows(codes, scales16, out, stream=None):
    rows, cols = codes.shape
    dt = QAT_DTYPE_BF16 if out.dtype == torch.bfloat16 else QAT_DTYPE_F32
    _check(lib().dequantize_rows(_p(codes), _p(scales16), rows, cols, dt, _p(out),
                                 _stream(stream)), "dequantize_rows")


def dequantize_rows_batch(items, stream=None):
    """items: list of (codes int8 [rows, cols], scales16 fp16 [rows], out fp32 or
    bf16 [rows, cols]) device tensors -- or an array from dequant_descs()."""
    arr = items if isinstance(items, ctypes.Array) else dequant_descs(items)
    _check(lib().dequantize_rows_batch(arr, len(arr), _stream(stream)), "dequantize_rows_batch")


def dequant_descs(items):
    """Marshal (codes, scales16, out) tuples into the C descriptor array once."""
    arr = (_DequantDesc * len(items))()
    for i, (codes, scales16, out) in enumerate(items):
        rows, cols = codes.shape
        dt = QAT_DTYPE_BF16 if out.dtype == torch.bfloat16 else QAT_DTYPE_F32
        arr[i] = _DequantDesc(codes.data_ptr(), scales16.data_ptr(), rows, cols, dt, 0, out.data_ptr())
    return arr


def qat_linear_fwd_noalloc(W, X, Y, bits, residual=None, ldx=0, T=None, stream=None):
    """The raw-weight QAT forward without workspace: for callers that cannot
    allocate device memory (its scratch is a fixed array inside the library)."""
    N, K = W.shape
    if T is None:
        T = X.shape[0]
    _check(lib().qat_linear_fwd_noalloc(_p(W), N, K, bits, _p(X), ldx, T, _p(residual), _p(Y),
                                        _stream(stream)), "qat_linear_fwd_noalloc")
