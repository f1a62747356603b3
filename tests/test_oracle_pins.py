"""Pins for the CPU oracle: what the pages and plain mathematics fix.

Each test ties the oracle to something other than itself: a worked example
printed on the pages (fixtures under tests/golden/, each with its source),
a closed form, exact rational arithmetic, brute force on tiny inputs, an
error bound, or an endpoint where the method reduces to a textbook GEMM.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _round_half_even(fr: Fraction) -> int:
    fl = math.floor(fr)
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def _exact_code(x, a, qmax=127):
    """Exact-rational reference code and whether it sits near a rounding tie."""
    if a == 0:
        return 0, False
    q = Fraction(float(x)) * qmax / Fraction(float(a))
    frac = q - math.floor(q)
    near_tie = abs(frac - Fraction(1, 2)) < Fraction(1, 2 ** 18) and frac != Fraction(1, 2)
    return max(-qmax, min(qmax, _round_half_even(q))), near_tie


# --------------------------------------------------------------------------
# Worked examples printed on the pages
# --------------------------------------------------------------------------
def test_scholia_int4_scale_example():
    g = _golden("scholia_int4_scale_example.json")
    x = np.array(g["x"], np.float32)
    q, a = oracle.quantize_per_tensor(x, g["qmax"])
    assert q.tolist() == g["closed_form_codes"]
    s = float(oracle.step_size(a, g["qmax"]))
    assert abs(s - g["printed"]["step"]) < 5e-5
    i = g["x"].index(g["printed"]["x"])
    assert q[i] == g["printed"]["q"]
    assert round(float(oracle.dequantize_codes(q[i], a, g["qmax"])), 3) == g["printed"]["x_hat"]


def test_scholia_outlier_example():
    g = _golden("scholia_outlier_example.json")
    x = np.array(g["x"], np.float32)
    q, a = oracle.quantize_per_tensor(x, g["qmax"])
    assert q.tolist() == g["printed"]["codes"]
    s = float(oracle.step_size(a, g["qmax"]))
    assert abs(s - g["printed"]["step"]) < 5e-4
    assert abs(0.21 / s - g["printed"]["ratio_of_0.21"]) < 5e-4


def test_tanjunchen_4096_split_example():
    g = _golden("tanjunchen_4096_split_example.json")
    H, d, v = g["hidden"], g["outlier_dim"], g["outlier_value"]
    rs = np.random.default_rng(0)
    x = np.where(rs.random(H) < 0.5, -1.0, 1.0) * g["background_magnitude"]
    x[d] = v
    X = x.astype(np.float16)[None, :]
    W = synth.make_weight(64, H, 0.02, seed=11)

    # No split (threshold = inf): one row, so per-row == per-tensor.
    r_inf = oracle.llm_int8_matmul(X, W, math.inf)
    s_inf = float(oracle.step_size(r_inf["x_scale"][0], 127))
    assert abs(s_inf - g["printed"]["per_tensor_step"]) < 5e-4
    bg = np.abs(r_inf["Xq"][0, np.arange(H) != d])
    lo, hi = g["printed"]["per_tensor_grid_points_for_background"]
    assert bg.min() >= lo and bg.max() <= hi
    assert r_inf["count"] == 0

    # Split at threshold 6: dim 2048 goes to the FP16 branch.
    r6 = oracle.llm_int8_matmul(X, W, g["threshold"])
    assert r6["count"] == 1 and r6["idx"].tolist() == [d]
    s6 = float(oracle.step_size(r6["x_scale"][0], 127))
    assert abs(s6 - g["printed"]["split_step"]) < 5e-5
    assert r6["Xq"][0, d] == 0
    assert set(np.abs(r6["Xq"][0, np.arange(H) != d]).tolist()) == {g["printed"]["split_grid"]}
    # The outlier dim is carried exactly: C_outlier = 70 * W[:, 2048].
    assert np.array_equal(r6["C_outlier"][0], v * W[:, d].astype(np.float64))
    # The activation codes are exact after the split (+-1 -> +-127 at step
    # 1/127), so what error is left comes from the weights; without the
    # split the +-1 entries land on +-2 at step 70/127 and the error grows.
    exact = X[0].astype(np.float64) @ W.astype(np.float64).T
    err6 = np.abs(r6["Y"][0].astype(np.float64) - exact).mean()
    errinf = np.abs(r_inf["Y"][0].astype(np.float64) - exact).mean()
    assert err6 < errinf / 5


# --------------------------------------------------------------------------
# Rounding: half to even (closed-form ties, exact in fp16 and fp32)
# --------------------------------------------------------------------------
def test_tie_break_half_to_even():
    a = 127.0 / 64.0                      # 1.984375, the row absmax
    row = np.array([[a, 65 / 128, 67 / 128, -65 / 128, -67 / 128]], np.float16)
    # 65/128*127/a = 32.5 exactly, 67/128*127/a = 33.5 exactly.
    Xq, xs = oracle.quantize_act_rows(row, np.zeros(5, bool))
    assert xs[0] == np.float32(a)
    assert Xq[0].tolist() == [127, 32, 34, -32, -34]


# --------------------------------------------------------------------------
# Detection by brute force, with the strict '>' reading
# --------------------------------------------------------------------------
def _brute_flags(X, thr):
    M, K = X.shape
    flags = [False] * K
    for j in range(K):
        for i in range(M):
            if abs(float(X[i, j])) > thr:
                flags[j] = True
    return flags


@pytest.mark.parametrize("K", [16, 48, 64, 80])
def test_detection_brute_force(K):
    rs = np.random.default_rng(K)
    X = (rs.standard_normal((5, K)) * 2).astype(np.float16)
    X[:, 3] = np.float16(0.5)
    X[2, 3] = np.float16(6.0)              # equal to the threshold: not an outlier
    X[:, 5] = np.float16(0.25)
    X[4, 5] = np.float16(6.00390625)       # next fp16 above 6: outlier
    X[:, 7] = np.float16(-0.5)
    X[1, 7] = np.float16(-7.0)             # negative side counts
    X[:, K - 1] = np.float16(9.0)          # last column (bitmap tail word)
    X[:, 9] = 0                            # all-zero column
    for thr in [6.0, 2.5, 0.0, math.inf]:
        mask, bitmap, count, idx = oracle.find_outlier_cols(X, thr)
        flags = _brute_flags(X, thr)
        assert mask.tolist() == flags
        assert count == sum(flags)
        assert idx.tolist() == [j for j in range(K) if flags[j]]
        assert bitmap.size == (K + 31) // 32
        for j in range(K):
            assert bool((int(bitmap[j // 32]) >> (j % 32)) & 1) == flags[j]
    m6, _, _, _ = oracle.find_outlier_cols(X, 6.0)
    assert not m6[3] and m6[5] and m6[7] and m6[K - 1]
    minf, _, cinf, _ = oracle.find_outlier_cols(X, math.inf)
    assert cinf == 0
    m0, _, _, _ = oracle.find_outlier_cols(X, 0.0)
    assert m0.tolist() == [bool(np.any(X[:, j] != 0)) for j in range(K)]


# --------------------------------------------------------------------------
# Quantisers against exact rational arithmetic
# --------------------------------------------------------------------------
def test_weight_quant_exact_rational():
    W = synth.make_weight(7, 40, 0.02, seed=3)
    W[3, :] = 0                            # all-zero row -> scale 0, codes 0
    Wq, aw = oracle.quantize_weight_rows(W)
    for n in range(W.shape[0]):
        a = max(abs(float(v)) for v in W[n])
        assert float(aw[n]) == a
        for k in range(W.shape[1]):
            q, near = _exact_code(W[n, k], a)
            if near:
                assert abs(int(Wq[n, k]) - q) <= 1
            else:
                assert int(Wq[n, k]) == q
    assert np.all(Wq[3] == 0) and aw[3] == 0
    nz = aw > 0
    assert np.all(np.abs(Wq[nz]).max(axis=1) == 127)


def test_act_quant_exact_rational_and_half_step_bound():
    X, _, cols = synth.random_case(9, 64, 4, 3, seed=12)
    X[4, :] = 0                                      # all-zero row
    mask, _, _, _ = oracle.find_outlier_cols(X, 6.0)
    assert mask.nonzero()[0].tolist() == cols.tolist()
    Xq, xs = oracle.quantize_act_rows(X, mask)
    for i in range(X.shape[0]):
        a = max([abs(float(X[i, j])) for j in range(X.shape[1]) if not mask[j]], default=0.0)
        assert float(xs[i]) == a
        for j in range(X.shape[1]):
            if mask[j]:
                assert Xq[i, j] == 0
                continue
            q, near = _exact_code(X[i, j], a)
            if near:
                assert abs(int(Xq[i, j]) - q) <= 1
            else:
                assert int(Xq[i, j]) == q
            if a > 0:  # rounding error at most half a step ([Scholia] s4: x_hat = s*q)
                assert abs(float(X[i, j]) - int(Xq[i, j]) * a / 127) <= a / 254 * (1 + 1e-6)
    assert np.all(Xq[4] == 0) and xs[4] == 0


def test_all_outlier_row_has_zero_scale():
    X = np.array([[7.0, 8.0], [0.5, -9.0]], np.float16)
    mask, _, _, _ = oracle.find_outlier_cols(X, 6.0)
    Xq, xs = oracle.quantize_act_rows(X, mask)
    assert mask.tolist() == [True, True]
    assert xs.tolist() == [0.0, 0.0] and np.all(Xq == 0)


# --------------------------------------------------------------------------
# INT32 GEMM: brute force, closed forms, overflow bound, orientation
# --------------------------------------------------------------------------
def test_int32_gemm_brute_force_nonsquare():
    rs = np.random.default_rng(5)
    Xq = rs.integers(-127, 128, size=(3, 64)).astype(np.int8)
    Wq = rs.integers(-127, 128, size=(5, 64)).astype(np.int8)
    C = oracle.int32_gemm(Xq, Wq)
    assert C.shape == (3, 5) and C.dtype == np.int32
    for i in range(3):
        for n in range(5):
            s = 0
            for k in range(64):
                s += int(Xq[i, k]) * int(Wq[n, k])
            assert int(C[i, n]) == s


def test_int32_gemm_closed_forms():
    K = 8192
    ones = np.full((2, K), 127, np.int8)
    C = oracle.int32_gemm(ones, np.full((3, K), 127, np.int8))
    assert np.all(C == 127 * 127 * K) and 127 * 127 * K == 132128768 < 2 ** 31 - 1
    alt = np.tile(np.array([127, -127], np.int8), K // 2)[None, :]
    assert np.all(oracle.int32_gemm(alt, np.full((1, K), 127, np.int8)) == 0)
    neg = oracle.int32_gemm(np.full((1, K), -127, np.int8), np.full((1, K), 127, np.int8))
    assert neg[0, 0] == -127 * 127 * K


def test_int32_gemm_skips_outlier_columns():
    # Zeroed codes at O make the full-K product equal the sum over non-O columns.
    X, W, cols = synth.random_case(6, 96, 5, 4, seed=13)
    r = oracle.llm_int8_matmul(X, W, 6.0)
    keep = ~r["mask"]
    for i in range(6):
        for n in range(5):
            s = sum(int(r["Xq"][i, k]) * int(r["Wq"][n, k]) for k in range(96) if keep[k])
            assert int(r["C"][i, n]) == s


# --------------------------------------------------------------------------
# Endpoints
# --------------------------------------------------------------------------
def test_threshold_inf_is_pure_vectorwise_int8():
    X, W, _ = synth.random_case(12, 128, 6, 3, seed=14)
    r = oracle.llm_int8_matmul(X, W, math.inf)
    assert r["count"] == 0
    assert np.array_equal(r["x_scale"], np.abs(X.astype(np.float32)).max(axis=1))
    # The fp16 weight enters only through outlier columns: replacing it changes nothing.
    W2 = (W.astype(np.float32) * 3 + 1).astype(np.float16)
    r2 = oracle.llm_int8_matmul(X, W2, math.inf, Wq=r["Wq"], w_scale=r["w_scale"])
    assert np.array_equal(r["Y"], r2["Y"])
    # Y is exactly the dequantised INT32 product (rounded once to fp16).
    ref = np.zeros((12, 6))
    for i in range(12):
        for n in range(6):
            c = sum(int(a) * int(b) for a, b in zip(r["Xq"][i], r["Wq"][n]))
            ref[i, n] = c * float(r["x_scale"][i]) * float(r["w_scale"][n]) / 16129.0
    assert np.array_equal(r["Y"], ref.astype(np.float16))


def test_threshold_zero_is_plain_fp16_gemm():
    X, W, _ = synth.random_case(4, 24, 3, 2, seed=15)
    X[:, 5] = 0
    r = oracle.llm_int8_matmul(X, W, 0.0)
    assert np.all(r["Xq"] == 0) and np.all(r["x_scale"] == 0)
    assert r["count"] == 23
    ref = np.zeros((4, 3))
    for i in range(4):
        for n in range(3):
            ref[i, n] = sum(float(X[i, k]) * float(W[n, k]) for k in range(24))
    assert np.allclose(r["Y"].astype(np.float64), ref.astype(np.float16).astype(np.float64), rtol=0, atol=0)


def test_threshold_zero_matches_library_gemm_larger():
    X, W, _ = synth.random_case(64, 256, 48, 5, seed=16)
    r = oracle.llm_int8_matmul(X, W, 0.0)
    ref = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    assert np.array_equal(r["Y"], ref)


# --------------------------------------------------------------------------
# Decomposition: rigorous error bound against the exact product
# --------------------------------------------------------------------------
def test_decomposition_error_bound():
    X, W, cols = synth.random_case(32, 256, 40, 4, seed=17)
    r = oracle.llm_int8_matmul(X, W, 6.0)
    assert r["idx"].tolist() == cols.tolist()
    X64 = X.astype(np.float64)
    W64 = W.astype(np.float64)
    exact = X64 @ W64.T
    keep = ~r["mask"]
    ax = r["x_scale"].astype(np.float64)
    aw = r["w_scale"].astype(np.float64)
    Xhat = r["Xq"].astype(np.float64) * ax[:, None] / 127
    # |x - x_hat| <= a/254 and |w - w_hat| <= aw/254 per element, so
    # |sum_{k not in O} (x w - x_hat w_hat)| <= sum (a/254 |w| + |x_hat| aw/254).
    bound = (ax[:, None] / 254) * (np.abs(W64[:, keep]).sum(axis=1))[None, :] \
        + (np.abs(Xhat[:, keep]).sum(axis=1))[:, None] * (aw[None, :] / 254)
    Y = r["Y"].astype(np.float64)
    fp16_half_ulp = np.abs(Y) * 2.0 ** -11 + 2.0 ** -25
    assert np.all(np.abs(Y - exact) <= bound * (1 + 1e-9) + fp16_half_ulp + 1e-12)
    # And the outlier split matters: per-row INT8 over every column is far worse.
    rinf = oracle.llm_int8_matmul(X, W, math.inf)
    err_mixed = np.abs(Y - exact).mean()
    err_inf = np.abs(rinf["Y"].astype(np.float64) - exact).mean()
    assert err_mixed < err_inf / 5


def test_sampled_outputs_match_full():
    X, W, _ = synth.random_case(40, 128, 24, 3, seed=18)
    r = oracle.llm_int8_matmul(X, W, 6.0)
    rs = np.random.default_rng(1)
    rows = rs.integers(0, 40, 50)
    cols = rs.integers(0, 24, 50)
    Ys, Cs, mask, xs = oracle.llm_int8_matmul_at(X, W, r["Wq"], r["w_scale"], 6.0, rows, cols)
    assert np.array_equal(Cs, r["C"][rows, cols])
    assert np.array_equal(xs, r["x_scale"][rows])
    assert np.array_equal(mask, r["mask"])
    assert np.allclose(Ys.astype(np.float64), r["Y"][rows, cols].astype(np.float64), rtol=1e-3, atol=1e-4)


def test_synthetic_outliers_detected_exactly():
    for name in ["tiny"]:
        w = synth.WORKLOADS[name]
        X, W, cols = synth.make_workload(w)
        _, _, count, idx = oracle.find_outlier_cols(X, w.threshold)
        assert idx.tolist() == cols.tolist() and count == w.n_outliers


# --------------------------------------------------------------------------
# The C++ oracle's plumbing: binary16 conversions against numpy's on every bit
# pattern and every rounding tie, the int32 overflow check, thread counts
# --------------------------------------------------------------------------
def test_half_decode_every_bit_pattern():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    got = oracle.half_to_float(h)
    ref = h.astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    # bit patterns, so that -0 and +0 are told apart
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_half_encode_values_ties_and_overflow():
    pos = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = (pos[:-1] + pos[1:]) / 2                  # exact ties between neighbours
    nxt = np.nextafter(mids, np.inf)
    prv = np.nextafter(mids, -np.inf)
    rs = np.random.default_rng(0)
    rnd = np.ldexp(rs.random(200000) + 0.5, rs.integers(-30, 18, 200000))
    edge = np.array([65504.0, 65519.99, 65520.0, 65536.0, 1e300, 2.0 ** -24, 2.0 ** -25,
                     np.nextafter(2.0 ** -25, 1), 2.0 ** -26, 0.0, np.inf])
    d = np.concatenate([pos, mids, nxt, prv, rnd, edge])
    d = np.concatenate([d, -d])
    got = oracle.double_to_half(d).view(np.uint16)
    ref = d.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    # ties go to the even significand
    t = oracle.double_to_half(mids).view(np.uint16)
    assert np.all(t % 2 == 0)


def test_int32_gemm_refuses_overflow():
    K = 133160                                       # 127^2 * K > 2^31 - 1
    with pytest.raises(AssertionError):
        oracle.int32_gemm(np.full((1, K), 127, np.int8), np.full((1, K), 127, np.int8))


def test_results_do_not_depend_on_thread_count():
    X, W, _ = synth.random_case(37, 256, 29, 5, seed=19)
    try:
        oracle.set_threads(1)
        r1 = oracle.llm_int8_matmul(X, W, 6.0)
        oracle.set_threads(7)
        r7 = oracle.llm_int8_matmul(X, W, 6.0)
    finally:
        oracle.set_threads(0)
    for key in ("Y", "mask", "idx", "Xq", "x_scale", "Wq", "w_scale", "C", "C_normal", "C_outlier"):
        assert np.array_equal(r1[key], r7[key]), key
