"""int8_mixed_matmul_noalloc: the matmul for callers that cannot give the library
device memory (for example code whose host framework owns every device
allocation, or code that must not grow its memory use while running).

The entry point keeps its scratch in a fixed device array inside the library.
This test calls it through the C ABI twice in a row, on different inputs, and
checks each result against the regular entry point (caller workspace) within
the Y tolerance used by the other GPU tests. It also checks that a problem too
large for the built-in array is refused. The file is named so that pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_TOL = 1e-2
MEAN_TOL = 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_quantized_matmul_b200 import _lib, build
    build.build()
    return _lib.load()


def _close(y, ref):
    y = y.astype(np.float64)
    ref = ref.astype(np.float64)
    d = np.abs(y - ref)
    assert np.all(np.isfinite(y))
    assert d.max() <= MAX_TOL * np.abs(ref).max() + 1e-6
    assert d.mean() <= MEAN_TOL * np.abs(ref).mean() + 1e-7


def test_noalloc_twice_in_a_row_matches_workspace_path(lib):
    from w8a8_quantized_matmul_b200 import _lib
    M, K, N = 300, 1024, 520
    X1, W, _ = synth.random_case(M, K, N, 6, seed=41)        # few outliers: epilogue path
    X2, _, _ = synth.random_case(M, K, N, 40, seed=42)       # many: tensor-core outlier pass
    Wd = torch.from_numpy(W).cuda()
    Wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty((N,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.int8_quantize_weight_rows(Wd.data_ptr(), N, K, Wq.data_ptr(), ws.data_ptr(), stream) == 0
    Xs = [torch.from_numpy(X1).cuda(), torch.from_numpy(X2).cuda()]

    # Regular entry point, caller-provided workspace.
    need = lib.int8_mixed_matmul_workspace_size(M, N, K)
    work = torch.empty((need,), dtype=torch.uint8, device="cuda")
    refs = []
    for Xd in Xs:
        Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        st = lib.int8_mixed_matmul(Xd.data_ptr(), Wq.data_ptr(), ws.data_ptr(), Wd.data_ptr(),
                                   M, N, K, 6.0, Y.data_ptr(), work.data_ptr(), need, stream)
        assert st == _lib.I8MM_OK
        refs.append(Y)

    # The allocation-free entry point, two calls back to back.
    outs = [torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda") for _ in Xs]
    for Xd, Y in zip(Xs, outs):
        st = lib.int8_mixed_matmul_noalloc(Xd.data_ptr(), Wq.data_ptr(), ws.data_ptr(),
                                           Wd.data_ptr(), M, N, K, 6.0, Y.data_ptr(), stream)
        assert st == _lib.I8MM_OK
    torch.cuda.synchronize()
    for Y, R in zip(outs, refs):
        _close(Y.cpu().numpy(), R.cpu().numpy())


def test_noalloc_refuses_problems_larger_than_its_array(lib):
    from w8a8_quantized_matmul_b200 import _lib
    # The OPT-6.7B FFN-up shape needs about 160 MB of scratch, more than the 64 MiB array;
    # the call is refused before anything is launched, so the pointers are never used.
    A = 1 << 20
    st = lib.int8_mixed_matmul_noalloc(A, A, A, A, 2048, 16384, 4096, 6.0, A, None)
    assert st == _lib.I8MM_ERR_WORKSPACE
