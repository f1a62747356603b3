"""Pins of the top-k decomposition in the oracle ([AIInfra] "05Quantization01",
LLM.int8() section, training notes: keep the top 1-2% largest-magnitude feature
dimensions in FP16 instead of a fixed threshold)."""
import numpy as np

import oracle
import synth


def test_brute_force_and_ties():
    X = np.array([[1.0, -5.0, 2.0, 5.0, 0.0, -3.0],
                  [0.5, 1.0, -4.0, 0.0, 0.0, 3.0]], np.float16)
    # column magnitudes: 1, 5, 4, 5, 0, 3 -> order 1, 3 (tie: lower index first), 2, 5, 0, 4
    expect = [[], [1], [1, 3], [1, 3, 2], [1, 3, 2, 5], [1, 3, 2, 5, 0], [0, 1, 2, 3, 4, 5]]
    for k, cols in enumerate(expect):
        mask = oracle.find_topk_cols(X, k)
        assert sorted(np.nonzero(mask)[0].tolist()) == sorted(cols)
    assert oracle.find_topk_cols(X, 99).all()
    assert not oracle.find_topk_cols(X, -3).any()


def test_planted_outliers_match_threshold_detection():
    for seed in range(3):
        X, W, cols = synth.random_case(128, 512, 16, 6, seed=100 + seed)
        mask = oracle.find_topk_cols(X, len(cols))
        np.testing.assert_array_equal(np.nonzero(mask)[0], np.sort(cols))
        np.testing.assert_array_equal(mask, oracle.find_outlier_cols(X, 6.0)[0])


def test_endpoints():
    X, W, _ = synth.random_case(32, 128, 24, 3, seed=7)
    Wq, ws = oracle.quantize_weight_rows(W)
    none = oracle.llm_int8_matmul(X, W, Wq=Wq, w_scale=ws, outlier_mask=oracle.find_topk_cols(X, 0))
    inf = oracle.llm_int8_matmul(X, W, float("inf"), Wq=Wq, w_scale=ws)
    np.testing.assert_array_equal(none["Y"], inf["Y"])
    allc = oracle.llm_int8_matmul(X, W, Wq=Wq, w_scale=ws, outlier_mask=oracle.find_topk_cols(X, 128))
    assert not allc["Xq"].any()
    exact = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    np.testing.assert_array_equal(allc["Y"], exact)
