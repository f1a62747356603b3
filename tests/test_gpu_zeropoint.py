"""Zero-point rows on the GPU against the oracle ([Scholia] "Inference
Quantization" notes, section 6; [AIInfra] "05Quantization01", LLM.int8()
section on one-sided outliers). Codes, steps, zero points, the outlier set and
the weight row sums are compared bit for bit, Y within the tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_quantized_matmul_b200 as m

pytestmark = pytest.mark.gpu


def wt(W):
    """The fp16 weight in the transposed [K][N] layout the mixed-matmul calls take."""
    return m.int8_transpose_weight(W)

MAX_REL, MEAN_REL = 1e-2, 1e-3


def _run(X, W, thr):
    M, K = X.shape
    N = W.shape[0]
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    rsum = m.int8_weight_rowsum(Wq)
    Y, work = m.int8_mixed_matmul_zp(Xd, Wq, ws, rsum, wt(Wd), thr)
    torch.cuda.synchronize()
    ref = oracle.llm_int8_matmul(X, W, thr, zeropoint=True)
    np.testing.assert_array_equal(rsum.cpu().numpy(), ref["wsum"])
    v = m.workspace_views(work, M, N, K)
    assert m.int8_device_status(work) == 0
    np.testing.assert_array_equal(v["col_bitmap"].cpu().numpy().view(np.uint32), ref["bitmap"])
    assert int(v["n_outliers"].item()) == ref["count"]
    np.testing.assert_array_equal(v["Xq"].cpu().numpy(), ref["Xq"])
    np.testing.assert_array_equal(v["x_scale"].cpu().numpy(), ref["x_scale"])
    np.testing.assert_array_equal(m.zeropoint_views(work, M, N, K).cpu().numpy(), ref["zero"])
    Yh = Y.cpu().numpy().astype(np.float64)
    Yr = ref["Y"].astype(np.float64)
    d = np.abs(Yh - Yr)
    assert d.max() <= MAX_REL * np.abs(Yr).max()
    assert d.mean() <= MEAN_REL * np.abs(Yr).mean()
    return Yh


CASES = [
    (256, 1024, 512, 6, 6.0),
    (300, 1040, 136, 3, 6.0),
    (2048, 4096, 1024, 6, 6.0),
    (256, 1024, 512, 40, 6.0),            # 40 outlier columns: one 64-column panel block
    (16, 512, 256, 2, 6.0),               # small M: single-CTA GEMM tiles
    (256, 1024, 512, 6, float("inf")),    # pure zero-point W8A8
    (128, 512, 256, 4, 0.0),              # every nonzero column an outlier
]


@pytest.mark.parametrize("case", CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}-o{c[3]}-t{c[4]}" for c in CASES])
def test_zeropoint_parity(case):
    M, K, N, n_out, thr = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=M + 3 * K + N)
    _run(X, W, thr)


def test_one_sided_rows():
    X, W, _ = synth.random_case(512, 1024, 256, 0, seed=4)
    X = np.abs(X).astype(np.float16)                 # every token non-negative
    Yz = _run(X, W, float("inf"))
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Ya, _ = m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), float("inf"))
    e_zp = np.abs(Yz - exact).mean()
    e_abs = np.abs(Ya.cpu().numpy().astype(np.float64) - exact).mean()
    assert e_zp < 0.8 * e_abs
