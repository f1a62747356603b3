"""Pins of the zero-point (asymmetric) per-token quantiser in the oracle.

[Scholia] "Inference Quantization" notes, section 6: q = clip(round(x/s) + z,
qmin, qmax), x_hat = s(q - z), z is the integer that represents real 0, and an
asymmetric grid covers data such as [-0.2, 1.7] with all of its levels.
[AIInfra] "05Quantization01", LLM.int8() section: the outliers are one-sided, so
zeropoint quantisation does better than absmax where they are not split off.
"""
import numpy as np

import oracle
import synth


def _row(values):
    x = np.array([values], np.float16)
    return x, np.zeros(x.shape[1], bool)


def test_section_6_range_uses_every_level_and_zero_is_exact():
    x, mask = _row(np.linspace(-0.2, 1.7, 97))
    x = np.concatenate([x, np.zeros((1, 1), np.float16)], axis=1)
    mask = np.zeros(x.shape[1], bool)
    q, step, zero = oracle.quantize_act_rows_zp(x, mask)
    assert q[0].min() == -128 and q[0].max() == 127          # both ends of the grid reached
    assert q[0, -1] == zero[0]                                 # real 0 is the integer z
    xh = step[0].astype(np.float64) * (q[0].astype(np.float64) - zero[0])
    assert np.max(np.abs(xh - x[0].astype(np.float64))) <= 0.5 * step[0] * (1 + 1e-6)


def test_one_sided_data_halves_the_step():
    rng = np.random.default_rng(3)
    x = np.abs(rng.standard_normal((1, 512))).astype(np.float16)
    mask = np.zeros(512, bool)
    _, step, zero = oracle.quantize_act_rows_zp(x, mask)
    a = float(np.max(x.astype(np.float32)))
    assert zero[0] == -128                                     # lo = 0 maps to the bottom
    assert abs(float(step[0]) - a / 255) <= 1e-7 * a
    # the symmetric absmax step for the same row is a / 127
    _, xs = oracle.quantize_act_rows(x, mask)
    assert abs(float(step[0]) / (float(xs[0]) / 127) - 127 / 255) < 1e-6


def test_outlier_columns_contribute_nothing_and_identity():
    X, W, cols = synth.random_case(24, 128, 16, 3, seed=5)
    mask = oracle.find_outlier_cols(X, 6.0)[0]
    Xq, step, zero = oracle.quantize_act_rows_zp(X, mask)
    assert (Xq[:, mask] == zero[:, None]).all()
    Wq, ws = oracle.quantize_weight_rows(W)
    C = oracle.int32_gemm(Xq, Wq)
    wsum = oracle.weight_rowsum(Wq)
    for i in range(24):
        for n in range(16):
            direct = sum((int(a) - int(zero[i])) * int(b) for a, b in zip(Xq[i], Wq[n]))
            assert direct == int(C[i, n]) - int(zero[i]) * int(wsum[n])


def test_brute_force_codes():
    X = np.array([[-1.5, 0.25, 3.0, 0.0], [2.0, 1.0, 0.5, 0.0], [0, 0, 0, 0]], np.float16)
    mask = np.array([False, False, False, True])
    q, step, zero = oracle.quantize_act_rows_zp(X, mask)
    for i in range(3):
        kept = [np.float32(v) for v, m in zip(X[i], mask) if not m]
        hi = max(np.float32(0), max(kept))
        lo = min(np.float32(0), min(kept))
        st = np.float32(np.float32(hi - lo) / np.float32(255))
        assert step[i] == st
        if st == 0:
            assert zero[i] == 0 and (q[i] == 0).all()
            continue
        z = int(np.clip(-128 - np.rint(np.float32(lo / st)), -128, 127))
        assert zero[i] == z
        for j in range(4):
            want = z if mask[j] else int(np.clip(np.rint(np.float32(np.float32(X[i, j]) / st)) + z, -128, 127))
            assert q[i, j] == want


def test_endpoints():
    X, W, _ = synth.random_case(32, 256, 24, 3, seed=8)
    allc = oracle.llm_int8_matmul(X, W, 0.0, zeropoint=True)
    assert not allc["Xq"].any()
    exact = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    nz = np.abs(X).max(axis=0) > 0
    if nz.all():
        np.testing.assert_array_equal(allc["Y"], exact)


def test_zeropoint_beats_absmax_on_one_sided_outliers_without_split():
    X, W, _ = synth.random_case(256, 512, 64, 6, seed=31, lo=20.0, hi=60.0)
    X = np.where(X < -6, -X, X).astype(np.float16)            # make every column's outliers positive
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    inf = float("inf")
    e_abs = np.abs(oracle.llm_int8_matmul(X, W, inf)["Y"] - exact).mean()
    e_zp = np.abs(oracle.llm_int8_matmul(X, W, inf, zeropoint=True)["Y"] - exact).mean()
    assert e_zp < 0.8 * e_abs
