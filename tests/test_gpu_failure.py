"""Failure reporting on the GPU without a fault: a bounded device wait that
nothing satisfies gives up after its limit, the kernel returns, the host reads
QAT_ERR_TIMEOUT from qat_device_error (which clears it), and the context keeps
working."""
import time

import numpy as np
import pytest
import torch

import oracle as o
from quantization_aware_tiny_b200 import qat

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    torch.cuda.synchronize()
    assert qat.device_error() == 0
    t0 = time.perf_counter()
    qat.qat_selftest_wait_timeout(20_000_000)  # 20 ms
    assert qat.device_error() == qat.QAT_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 5.0, elapsed  # it waited about its limit, then returned
    assert qat.device_error() == 0  # read once, then cleared
    # the context still runs the library's kernels correctly
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    q = qat.quantize_weight(torch.from_numpy(W).cuda(), 6, keep_codes=True)
    torch.cuda.synchronize()
    assert np.array_equal(q.codes.cpu().numpy(), o.quantize_weight(W, 6)["codes"])
    assert qat.device_error() == 0
