"""Top-k decomposition on the GPU against the oracle ([AIInfra] "05Quantization01",
LLM.int8() section, training notes: the top 1-2% largest-magnitude feature
dimensions in FP16). The selected set (bitmap, count, list), the codes and the
scales are compared bit for bit, Y within the tolerance."""
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


def _check(X, W, k):
    M, K = X.shape
    N = W.shape[0]
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y, work = m.int8_mixed_matmul_topk(Xd, Wq, ws, wt(Wd), k)
    torch.cuda.synchronize()
    mask = oracle.find_topk_cols(X, k)
    ref = oracle.llm_int8_matmul(X, W, outlier_mask=mask)
    v = m.workspace_views(work, M, N, K)
    assert m.int8_device_status(work) == 0
    np.testing.assert_array_equal(v["col_bitmap"].cpu().numpy().view(np.uint32), ref["bitmap"])
    assert int(v["n_outliers"].item()) == ref["count"]
    np.testing.assert_array_equal(v["col_idx"].cpu().numpy()[:ref["count"]], ref["idx"])
    np.testing.assert_array_equal(v["Xq"].cpu().numpy(), ref["Xq"])
    np.testing.assert_array_equal(v["x_scale"].cpu().numpy(), ref["x_scale"])
    Yh = Y.cpu().numpy().astype(np.float64)
    Yr = ref["Y"].astype(np.float64)
    d = np.abs(Yh - Yr)
    assert d.max() <= MAX_REL * np.abs(Yr).max()
    assert d.mean() <= MEAN_REL * np.abs(Yr).mean()
    return Y


@pytest.mark.parametrize("k", [0, 1, 6, 41, 82, 4095, 4096])
def test_topk_parity_opt_like(k):
    X, W, _ = synth.random_case(256, 4096, 384, 6, seed=501)
    _check(X, W, k)


# K up to 8192 takes the rank select, larger K the one-CTA radix select: both sides of the switch.
@pytest.mark.parametrize("case", [(300, 1040, 136, 3, 10), (17, 512, 200, 2, 5), (129, 272, 264, 0, 3),
                                  (40, 8192, 136, 4, 82), (40, 8208, 136, 4, 82),
                                  (40, 20480, 136, 0, 400)])
def test_topk_parity_shapes(case):
    M, K, N, n_out, k = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=M + K + N)
    _check(X, W, k)


def test_topk_ties_go_to_lower_index():
    X, W, _ = synth.random_case(64, 512, 128, 0, seed=9)
    X[:, :] = np.clip(X, -1.0, 1.0)
    X[0, 100:140] = 3.0          # 40 columns tied at the largest magnitude
    _check(X, W, 10)             # the ten lowest of them: 100..109
    mask = oracle.find_topk_cols(X, 10)
    assert np.nonzero(mask)[0].tolist() == list(range(100, 110))


def test_k0_equals_threshold_inf():
    X, W, _ = synth.random_case(512, 1024, 256, 6, seed=12)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Yk, _ = m.int8_mixed_matmul_topk(Xd, Wq, ws, wt(Wd), 0)
    Yi, _ = m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), float("inf"))
    assert torch.equal(Yk, Yi)


def test_topk_ties_go_to_lower_index_radix_select():
    X, W, _ = synth.random_case(32, 20480, 128, 0, seed=19)
    X[:, :] = np.clip(X, -1.0, 1.0)
    X[1, 18000:18100] = 3.0      # 100 tied columns, high in K
    X[2, 50:60] = 3.0            # 10 more, low in K
    _check(X, W, 30)             # 50..59, then 18000..18019
    mask = oracle.find_topk_cols(X, 30)
    assert np.nonzero(mask)[0].tolist() == list(range(50, 60)) + list(range(18000, 18020))
