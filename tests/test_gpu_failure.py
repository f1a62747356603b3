"""Failure detection without a GPU fault: a device-side wait on a phase that
nothing completes gives up after its bound, records I8MM_ERR_TIMEOUT and lets
the kernel exit; the context stays usable for the next call."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_quantized_matmul_b200 as m
from w8a8_quantized_matmul_b200 import _lib

pytestmark = pytest.mark.gpu


def wt(W):
    """The fp16 weight in the transposed [K][N] layout the mixed-matmul calls take."""
    return m.int8_transpose_weight(W)


def test_bounded_wait_reports_timeout_and_context_survives():
    assert m.selftest_wait_timeout() == _lib.I8MM_ERR_TIMEOUT
    # the next call on the same context runs normally
    X, W, _ = synth.random_case(32, 256, 64, 2, seed=77)
    Wq, ws = m.int8_quantize_weight_rows(torch.from_numpy(W).cuda())
    Y, work = m.int8_mixed_matmul(torch.from_numpy(X).cuda(), Wq, ws, wt(torch.from_numpy(W).cuda()))
    torch.cuda.synchronize()
    assert m.int8_device_status(work) == 0
    ref = oracle.llm_int8_matmul(X, W, 6.0)["Y"].astype(np.float64)
    d = np.abs(Y.cpu().numpy().astype(np.float64) - ref)
    assert d.max() <= 1e-2 * np.abs(ref).max()
