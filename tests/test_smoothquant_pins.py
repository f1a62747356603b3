"""Pins of the SmoothQuant oracle (oracle/smoothquant.py) against the pages and
the mathematics ([Tanjunchen] "quantization explained part 2", section 4).

- section 4.5 worked example: the printed mean output errors of per-tensor
  W8A8 before and after smoothing (0.108 -> 0.054, alpha = 0.5), with the
  example's inputs redrawn from the same seed and order;
- section 4.2 equivalence: X diag(s)^-1 . diag(s) W = X W exactly (float64);
- closed forms of the factors at alpha = 0, 0.5, 1 and for empty channels;
- alpha = 1 calibrated on X itself makes every channel's max |X_hat| = 1;
- brute force of the runtime quantiser and INT32 product on tiny inputs;
- smoothing lowers the W8A8 error when the activations have outlier channels.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "tanjunchen_smoothquant_example.json")


def _example_inputs(g):
    torch.manual_seed(0)
    X = torch.randn(g["tokens"], g["in_channels"])
    X[:, g["outlier_channel"]] *= g["outlier_scale"]
    W_in_out = torch.randn(g["in_channels"], g["out_channels"]) * g["weight_std"]
    return X.double().numpy(), W_in_out.double().numpy().T.copy()   # our W is [out][in]


def test_section_4_5_example_errors():
    g = json.load(open(GOLDEN))
    X, W = _example_inputs(g)
    Y = X @ W.T
    pq = oracle.per_tensor_quant_dequant
    err_raw = np.abs(Y - pq(X) @ pq(W).T).mean()
    s = oracle.smooth_factors(oracle.column_absmax(X), W, g["alpha"])
    X_hat = X / s[None, :]
    W_hat = W * s[None, :]
    err_smooth = np.abs(Y - pq(X_hat) @ pq(W_hat).T).mean()
    d = g["printed_decimals"]
    assert round(err_raw, d) == g["mean_abs_error_unsmoothed"]
    assert round(err_smooth, d) == g["mean_abs_error_smoothed"]
    # section 4.5: the equivalence error is round-off only (~1e-6 in fp32)
    assert np.abs(X_hat @ W_hat.T - Y).max() < 1e-12 * max(1.0, np.abs(Y).max())


def test_equivalence_random():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((40, 24))
    X[:, 7] *= 50
    W = 0.02 * rng.standard_normal((10, 24))
    for alpha in (0.0, 0.3, 0.5, 0.8, 1.0):
        s = oracle.smooth_factors(oracle.column_absmax(X), W, alpha)
        lhs = (X / s[None, :]) @ (W * s[None, :]).T
        np.testing.assert_allclose(lhs, X @ W.T, rtol=1e-12, atol=1e-12)


def test_factor_closed_forms():
    act = np.array([4.0, 9.0, 0.0, 2.0, 1.0], np.float32)
    W = np.array([[1.0, -0.5, 3.0, 0.0, 2.0],
                  [-4.0, 0.25, 1.0, 0.0, -1.0]], np.float16)
    wmax = np.array([4.0, 0.5, 3.0, 0.0, 2.0])
    s = oracle.smooth_factors(act, W, 0.5)
    np.testing.assert_allclose(s[[0, 1, 4]], np.sqrt(act[[0, 1, 4]] / wmax[[0, 1, 4]]), rtol=1e-15)
    assert s[2] == 1.0 and s[3] == 1.0           # empty activation / weight channel
    np.testing.assert_allclose(oracle.smooth_factors(act, W, 1.0)[[0, 1, 4]], act[[0, 1, 4]])
    np.testing.assert_allclose(oracle.smooth_factors(act, W, 0.0)[[0, 1, 4]], 1.0 / wmax[[0, 1, 4]])


def test_alpha_one_flattens_channels():
    X, _, _ = synth.random_case(64, 96, 8, 4, seed=3)
    W = np.ones((4, 96), np.float16)
    s32 = oracle.smooth_factors(oracle.column_absmax(X), W, 1.0).astype(np.float32)
    r = oracle.smooth_rcp(s32)
    _, _, X_hat = oracle.smooth_act_rows(X, r)
    colmax = np.abs(X_hat).max(axis=0)
    live = oracle.column_absmax(X) > 0
    np.testing.assert_allclose(colmax[live], 1.0, rtol=2 ** -22)


def test_runtime_quantiser_brute_force():
    X = np.array([[0.5, -3.0, 1.25], [0.0, 0.0, 0.0], [7.0, 0.1, -7.5]], np.float16)
    r = np.array([2.0, 0.5, 0.3], np.float32)
    Xq, xs, X_hat = oracle.smooth_act_rows(X, r)
    for i in range(3):
        xh = [np.float32(np.float32(X[i, j]) * r[j]) for j in range(3)]
        a = max(abs(v) for v in xh)
        assert xs[i] == np.float32(a)
        for j in range(3):
            want = 0 if a == 0 else int(np.clip(np.rint(np.float32(xh[j] * np.float32(127)) / np.float32(a)), -127, 127))
            assert Xq[i, j] == want


def test_matmul_brute_force():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((5, 32)).astype(np.float16)
    W = (0.05 * rng.standard_normal((3, 32))).astype(np.float16)
    s32 = oracle.smooth_factors(oracle.column_absmax(X), W, 0.5).astype(np.float32)
    Wq, ws, _ = oracle.smooth_weight_rows(W, s32)
    out = oracle.smoothquant_matmul(X, Wq, ws, oracle.smooth_rcp(s32))
    for i in range(5):
        for n in range(3):
            c = sum(int(a) * int(b) for a, b in zip(out["Xq"][i], Wq[n]))
            assert out["C"][i, n] == c
            y = np.float16(c * float(out["x_scale"][i]) * float(ws[n]) / 16129.0)
            assert out["Y"][i, n] == y


def test_smoothing_lowers_w8a8_error_with_outlier_channels():
    X, W, _ = synth.random_case(256, 512, 64, 6, seed=21)
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    ones = np.ones(512, np.float32)
    Wq0, ws0, _ = oracle.smooth_weight_rows(W, ones)
    e0 = np.abs(oracle.smoothquant_matmul(X, Wq0, ws0, ones)["Y"] - Y).mean()
    s32 = oracle.smooth_factors(oracle.column_absmax(X), W, 0.5).astype(np.float32)
    Wq, ws, _ = oracle.smooth_weight_rows(W, s32)
    e1 = np.abs(oracle.smoothquant_matmul(X, Wq, ws, oracle.smooth_rcp(s32))["Y"] - Y).mean()
    assert e1 < 0.7 * e0
