"""int8_mixed_matmul_noalloc: the matmul for callers that cannot give the library
device memory (for example code whose host framework owns every device
allocation and hands it no allocator, or code that must not grow its memory use
while running).

The entry point keeps its scratch in a fixed device array inside the library.
These tests call it through the C ABI twice in a row, on different inputs, at a
prefill shape (few outliers: the product in the GEMM epilogue; many: the
tensor-core outlier pass) and at a decode shape (16 tokens: the clustered decode
kernel; with 6 outlier columns and with none). The same kernels run as for the
regular entry point with a caller workspace, on the same inputs, so each result
must equal that entry point's bit for bit (which is within the Y tolerance of
the other GPU tests); the first result of each pair is also checked against the
CPU oracle within that tolerance. After the calls the status word of the
built-in array must read I8MM_OK. A problem too large for the array is refused.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import oracle
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


def _pair(lib, M, K, N, cases):
    """Two back-to-back no-alloc calls compared with the workspace entry point."""
    from w8a8_quantized_matmul_b200 import _lib
    Xs_h = []
    W = None
    for n_out, seed in cases:
        X, Wc, _ = synth.random_case(M, K, N, n_out, seed=seed)
        Xs_h.append(X)
        W = Wc if W is None else W
    Wd = torch.from_numpy(W).cuda()
    Wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty((N,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.int8_quantize_weight_rows(Wd.data_ptr(), N, K, Wq.data_ptr(), ws.data_ptr(),
                                         stream) == 0
    # The mixed-matmul calls take the fp16 weight transposed, [K][N].
    Wt = torch.empty((K, N), dtype=torch.float16, device="cuda")
    assert lib.int8_transpose_weight(Wd.data_ptr(), N, K, Wt.data_ptr(), stream) == 0
    Xs = [torch.from_numpy(X).cuda() for X in Xs_h]

    # Regular entry point, caller-provided workspace.
    need = lib.int8_mixed_matmul_workspace_size(M, N, K)
    work = torch.empty((need,), dtype=torch.uint8, device="cuda")
    refs = []
    for Xd in Xs:
        Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        st = lib.int8_mixed_matmul(Xd.data_ptr(), Wq.data_ptr(), ws.data_ptr(), Wt.data_ptr(),
                                   M, N, K, 6.0, Y.data_ptr(), work.data_ptr(), need, stream)
        assert st == _lib.I8MM_OK
        refs.append(Y)

    # The allocation-free entry point, two calls back to back.
    outs = [torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda") for _ in Xs]
    for Xd, Y in zip(Xs, outs):
        st = lib.int8_mixed_matmul_noalloc(Xd.data_ptr(), Wq.data_ptr(), ws.data_ptr(),
                                           Wt.data_ptr(), M, N, K, 6.0, Y.data_ptr(), stream)
        assert st == _lib.I8MM_OK
    assert lib.int8_noalloc_device_status(stream) == _lib.I8MM_OK
    torch.cuda.synchronize()
    for Y, R in zip(outs, refs):
        assert torch.equal(Y, R)
        _close(Y.cpu().numpy(), R.cpu().numpy())
    r = oracle.llm_int8_matmul(Xs_h[0], W, 6.0, Wq=Wq.cpu().numpy(), w_scale=ws.cpu().numpy(),
                               intermediates=False)
    _close(outs[0].cpu().numpy(), r["Y"])


def test_noalloc_prefill_twice_in_a_row_matches_workspace_path(lib):
    # 6 outlier columns: the product in the GEMM epilogue; 40: the tensor-core pass.
    _pair(lib, 300, 1024, 520, [(6, 41), (40, 42)])


def test_noalloc_decode_shape_twice_in_a_row_matches_workspace_path(lib):
    # 16 tokens: the clustered decode kernel; 6 outlier columns, then none.
    _pair(lib, 16, 4096, 520, [(6, 43), (0, 44)])


def test_noalloc_refuses_problems_larger_than_its_array(lib):
    from w8a8_quantized_matmul_b200 import _lib
    # The OPT-6.7B FFN-up shape needs about 160 MB of scratch, more than the 64 MiB array;
    # the call is refused before anything is launched, so the pointers are never used.
    A = 1 << 20
    st = lib.int8_mixed_matmul_noalloc(A, A, A, A, 2048, 16384, 4096, 6.0, A, None)
    assert st == _lib.I8MM_ERR_WORKSPACE
