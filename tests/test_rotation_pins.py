"""Pins of the grouped Hadamard rotation oracle (W8A8 and W4A4 after rotation).

[Baidu] developer.baidu.com "分组旋转方法从W8A8到W4A4": section 2 (an orthogonal,
regular Hadamard transform per group before quantisation), section 5.1 (G x G
sub-blocks, per sub-block parameters, packed 4-bit integers), section 5.2
(activation sub-blocks rotated then quantised), section 5.4 (eight 4-bit
integers per 32-bit word, INT32 accumulation, dequantisation).
[Scholia] "Inference Quantization" notes, section 4: the symmetric INT4 grid.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fp16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _outlier_acts(rng, M, K, n_out=6, mag=40.0):
    X = rng.standard_normal((M, K)) * 0.5
    cols = rng.choice(K, n_out, replace=False)
    X[:, cols] *= mag
    return X.astype(np.float16)


# ------------------------------------------------------------------ the matrix
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_sylvester_matrix_matches_library(G):
    assert np.array_equal(oracle.hadamard(G), scipy.linalg.hadamard(G))


@pytest.mark.parametrize("G", [16, 128])
def test_entry_closed_form_and_orthogonality(G):
    H = oracle.hadamard(G)
    i = np.arange(G)[:, None]
    j = np.arange(G)[None, :]
    parity = np.vectorize(lambda v: bin(int(v)).count("1") & 1)(i & j)
    assert np.array_equal(H, 1 - 2 * parity)              # H[i, j] = (-1)^popcount(i & j)
    assert np.array_equal(H @ H.T, G * np.eye(G, dtype=np.int64))


def test_non_power_of_two_rejected():
    with pytest.raises(ValueError):
        oracle.hadamard(12)
    with pytest.raises(ValueError):
        oracle.rotate_groups(np.zeros((1, 96), np.float16), 64)


@pytest.mark.parametrize("G", [16, 64, 128, 256])
def test_normalisation_is_the_nearest_fp32_to_inverse_root(G):
    c = oracle.rotation_scale(G)
    assert c.dtype == np.float32
    lo = np.nextafter(c, np.float32(0))
    hi = np.nextafter(c, np.float32(1))
    # 1/sqrt(G) lies between the midpoints (lo+c)/2 and (c+hi)/2: compare squares with 1/G
    m_lo = (Fraction(float(lo)) + Fraction(float(c))) / 2
    m_hi = (Fraction(float(c)) + Fraction(float(hi))) / 2
    assert m_lo * m_lo <= Fraction(1, G) <= m_hi * m_hi
    k = G.bit_length() - 1
    if k % 2 == 0:
        assert float(c) == 2.0 ** (-k // 2)


# ------------------------------------------------------------------ the rotation
def test_sums_are_exact_brute_force():
    rng = np.random.default_rng(11)
    # wide dynamic range: subnormal-ish to large fp16 values in the same group
    X = (rng.standard_normal((3, 32)) * np.exp2(rng.integers(-20, 14, (3, 32)))).astype(np.float16)
    G = 16
    S = oracle.hadamard_sums(X, G)
    for r in range(3):
        for g in range(32 // G):
            for i in range(G):
                exact = sum((Fraction(float(X[r, g * G + j])) *
                             (-1 if bin(i & j).count("1") & 1 else 1)) for j in range(G))
                assert Fraction(float(S[r, g * G + i])) == exact


def test_rotated_value_rounds_the_exact_sum_then_scales():
    rng = np.random.default_rng(5)
    X = _fp16(rng, (4, 256))
    for G in (64, 128):
        r = oracle.rotate_groups(X, G)
        S = oracle.hadamard_sums(X, G)
        c = oracle.rotation_scale(G)
        for (a, b) in [(0, 0), (1, 77), (3, 255), (2, 130)]:
            s32 = np.float32(S[a, b])                       # one rounding of the exact sum
            assert abs(Fraction(float(s32)) - Fraction(float(S[a, b]))) <= abs(Fraction(float(np.spacing(s32)))) / 2
            assert r[a, b] == np.float32(s32 * c)
        # every entry: the exact sum is rounded to fp32 BEFORE the scaling
        assert np.array_equal(r, S.astype(np.float32) * c)
        if G == 128:
            assert not np.array_equal(r, (S * float(c)).astype(np.float32))


def test_spike_spreads_evenly_over_its_group():
    G, K = 128, 512
    v = np.float16(24.0)
    for j in (0, 5, 127 + 128 * 2):
        x = np.zeros((1, K), np.float16)
        x[0, j] = v
        r = oracle.rotate_groups_f64(x, G)[0]
        g = j // G
        grp = r[g * G:(g + 1) * G]
        jj = j - g * G
        signs = np.array([1 - 2 * (bin(jj & i).count("1") & 1) for i in range(G)])
        assert np.allclose(grp, signs * float(v) / np.sqrt(G), rtol=0, atol=1e-12)
        assert np.all(np.delete(r, np.arange(g * G, (g + 1) * G)) == 0)
        assert np.max(np.abs(grp)) * np.sqrt(G) == pytest.approx(float(v))


def test_constant_group_collapses_to_first_entry():
    G = 64
    x = np.full((1, 2 * G), np.float16(0.75))
    r = oracle.rotate_groups_f64(x, G)[0]
    for g in range(2):
        assert r[g * G] == pytest.approx(0.75 * np.sqrt(G), abs=1e-12)
        assert np.all(r[g * G + 1:(g + 1) * G] == 0)


@pytest.mark.parametrize("G", [16, 128, 256])
def test_product_and_norms_preserved(G):
    rng = np.random.default_rng(7)
    X = _outlier_acts(rng, 8, 512)
    W = _fp16(rng, (6, 512), 0.05)
    XR = oracle.rotate_groups_f64(X, G)
    WR = oracle.rotate_groups_f64(W, G)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.max(np.abs(XR @ WR.T - ref)) <= 1e-10 * np.max(np.abs(ref))
    n0 = np.linalg.norm(X.astype(np.float64).reshape(8, -1, G), axis=2)
    n1 = np.linalg.norm(XR.reshape(8, -1, G), axis=2)
    assert np.allclose(n0, n1, rtol=1e-12, atol=0)
    # the rotation is its own inverse (symmetric and orthogonal)
    back = oracle.rotate_groups_f64(XR, G)
    assert np.allclose(back, X.astype(np.float64), rtol=0, atol=1e-9)
    # the fp32 values are within two roundings of the float64 ones
    r32 = oracle.rotate_groups(X, G).astype(np.float64)
    assert np.all(np.abs(r32 - XR) <= 2 * 2.0 ** -23 * np.abs(XR) + 1e-30)


def test_rotation_acts_along_k_only():
    """Rotating along the other axis would not preserve X W^T; a row's result
    depends only on that row."""
    rng = np.random.default_rng(9)
    X = _fp16(rng, (4, 128))
    r_all = oracle.rotate_groups(X, 32)
    for i in range(4):
        assert np.array_equal(oracle.rotate_groups(X[i:i + 1], 32)[0], r_all[i])


# ------------------------------------------------------------------ W8A8
def test_w8a8_rows_brute_force_and_bound():
    rng = np.random.default_rng(13)
    M, N, K, G = 3, 5, 64, 16
    X = _outlier_acts(rng, M, K, n_out=2, mag=20)
    W = _fp16(rng, (N, K), 0.1)
    Wq, aw, WR = oracle.quantize_rows_rotated(W, G)
    out = oracle.rotated_w8a8_matmul(X, Wq, aw, G)
    Xq, ax, XR = out["Xq"], out["x_scale"], out["R"]
    assert np.max(np.abs(Xq.astype(int))) == 127
    for m in range(M):
        assert ax[m] == np.max(np.abs(XR[m]))
        for n in range(N):
            c = sum(int(Xq[m, k]) * int(Wq[n, k]) for k in range(K))
            assert out["C"][m, n] == c
            y = c * float(ax[m]) * float(aw[n]) / (127 * 127)
            assert float(out["Y"][m, n]) == float(np.float16(y))
    # each code is within half a step of the rotated value, so Y is within the
    # propagated half-step bound of X W^T
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    ex = ax.astype(np.float64) / 254
    ew = aw.astype(np.float64) / 254
    bound = (np.abs(XR).astype(np.float64) @ np.broadcast_to(ew[:, None], (N, K)).T
             + ex[:, None] * np.abs(WR).astype(np.float64).sum(axis=1)[None, :]
             + K * ex[:, None] * ew[None, :]) * (1 + 1e-5) + 1e-3 * np.abs(ref)
    assert np.all(np.abs(out["Y"].astype(np.float64) - ref) <= bound + 1e-3)


def test_w8a8_rotation_lowers_error_on_outlier_channels():
    rng = np.random.default_rng(17)
    M, N, K, G = 32, 48, 1024, 128
    X = _outlier_acts(rng, M, K, n_out=8, mag=60)
    W = _fp16(rng, (N, K), 0.05)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    Wq, aw, _ = oracle.quantize_rows_rotated(W, G)
    Yr = oracle.rotated_w8a8_matmul(X, Wq, aw, G)["Y"].astype(np.float64)
    # the same per-token / per-row scheme without rotation
    Xq0, ax0 = oracle.quantize_act_rows(X, np.zeros(K, bool))
    Wq0, aw0 = oracle.quantize_weight_rows(W)
    Y0 = oracle.dequantize(oracle.int32_gemm(Xq0, Wq0), ax0, aw0)
    e_rot = np.mean(np.abs(Yr - ref))
    e_plain = np.mean(np.abs(Y0 - ref))
    assert e_rot < 0.5 * e_plain


# ------------------------------------------------------------------ W4A4
def test_int4_grid_of_the_scholia_example():
    g = json.load(open(os.path.join(GOLDEN, "scholia_int4_scale_example.json")))
    x = np.array(g["x"], np.float32)
    q = oracle.absmax_codes(x, np.float32(np.max(np.abs(x))), oracle.QMAX_W4)
    assert oracle.QMAX_W4 == g["qmax"]
    assert q.tolist() == g["closed_form_codes"]


def test_pack_word_layout():
    q = np.array([[1, -1, 2, -2, 3, -3, 7, -7, 0, 0, 0, 0, 0, 0, 0, -8]], np.int8)
    p = oracle.pack_int4(q)
    assert p.dtype == np.uint32 and p.shape == (1, 2)
    assert int(p[0, 0]) == 0x97D3E2F1
    assert int(p[0, 1]) == 0x80000000
    assert np.array_equal(oracle.unpack_int4(p), q)
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, (5, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(q)), q)
    with pytest.raises(ValueError):
        oracle.pack_int4(np.array([[8, 0, 0, 0, 0, 0, 0, 0]]))


def test_group_scales_brute_force():
    rng = np.random.default_rng(19)
    G, M, N, K = 16, 3, 32, 48
    X = _outlier_acts(rng, M, K, n_out=2, mag=10)
    W = _fp16(rng, (N, K), 0.2)
    Xq, ax, XR = oracle.quantize_act_groups(X, G)
    Wq, aw, WR = oracle.quantize_weight_blocks(W, G)
    assert ax.shape == (M, K // G) and aw.shape == (N // G, K // G)
    for m in range(M):
        for g in range(K // G):
            assert ax[m, g] == max(abs(float(v)) for v in XR[m, g * G:(g + 1) * G])
    for b in range(N // G):
        for g in range(K // G):
            blk = WR[b * G:(b + 1) * G, g * G:(g + 1) * G]
            assert aw[b, g] == max(abs(float(v)) for v in blk.ravel())
    assert np.all(np.abs(Xq.astype(int)) <= 7) and np.all(np.abs(Wq.astype(int)) <= 7)
    # every group that is not all zero reaches the end of the grid
    for m in range(M):
        for g in range(K // G):
            assert np.max(np.abs(Xq[m, g * G:(g + 1) * G].astype(int))) == 7
    # dequantised Y by plain loops over k
    out = oracle.rotated_w4a4_matmul(X, oracle.pack_int4(Wq), aw, G)
    assert np.array_equal(out["Xq"], Xq)
    for m in range(M):
        for n in range(N):
            y = sum(int(Xq[m, k]) * int(Wq[n, k]) * float(ax[m, k // G]) * float(aw[n // G, k // G])
                    for k in range(K)) / 49.0
            assert abs(float(out["Y"][m, n]) - y) <= 1e-3 * abs(y) + 1e-6
    # the group products add up to the whole product
    assert np.array_equal(out["Cg"].astype(np.int64).sum(axis=0),
                          oracle.int32_gemm(Xq, Wq).astype(np.int64))


def test_group_dequant_reduces_to_row_dequant_with_equal_scales():
    rng = np.random.default_rng(23)
    G, M, N, K = 16, 4, 32, 64
    Xq = rng.integers(-7, 8, (M, K)).astype(np.int8)
    Wq = rng.integers(-7, 8, (N, K)).astype(np.int8)
    ax_row = rng.uniform(0.5, 2, M).astype(np.float32)
    aw_row = rng.uniform(0.5, 2, N // G).astype(np.float32)
    ax = np.repeat(ax_row[:, None], K // G, axis=1)
    aw = np.repeat(aw_row[:, None], K // G, axis=1)
    Yg = oracle.dequantize_groups(oracle.group_gemm(Xq, Wq, G), ax, aw, G, 7)
    C = oracle.int32_gemm(Xq, Wq).astype(np.float64)
    Yr = C * ax_row[:, None] * np.repeat(aw_row, G)[None, :] / 49.0
    assert np.allclose(Yg, Yr, rtol=1e-12, atol=0)


def test_w4a4_rotation_lowers_error_on_outlier_channels():
    rng = np.random.default_rng(29)
    M, N, K, G = 16, 128, 1024, 128
    X = _outlier_acts(rng, M, K, n_out=8, mag=60)
    W = _fp16(rng, (N, K), 0.05)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    Wq, aw, _ = oracle.quantize_weight_blocks(W, G)
    Yr = oracle.rotated_w4a4_matmul(X, oracle.pack_int4(Wq), aw, G)["Y"].astype(np.float64)
    # the same sub-block scheme with the identity in place of the rotation
    X32 = X.astype(np.float32)
    ax0 = np.abs(X32).reshape(M, K // G, G).max(axis=2)
    Xq0 = oracle.absmax_codes(X32, np.repeat(ax0, G, axis=1), 7)
    W32 = W.astype(np.float32)
    aw0 = np.abs(W32).reshape(N // G, G, K // G, G).max(axis=(1, 3))
    Wq0 = oracle.absmax_codes(W32, np.repeat(np.repeat(aw0, G, 0), G, 1), 7)
    Y0 = oracle.dequantize_groups(oracle.group_gemm(Xq0, Wq0, G), ax0, aw0, G, 7)
    # the 4-bit weight error is common to both, so the gain in Y is smaller
    # than in the activations (about 0.8 here)
    assert np.mean(np.abs(Yr - ref)) < 0.9 * np.mean(np.abs(Y0 - ref))
    # the activations themselves, rotated back: the error falls by more than half
    Xq, ax, _ = oracle.quantize_act_groups(X, G)
    back = oracle.rotate_groups_f64(Xq.astype(np.float64) * np.repeat(ax, G, axis=1) / 7, G)
    e_rot = np.mean(np.abs(back - X.astype(np.float64)))
    e_plain = np.mean(np.abs(Xq0 * np.repeat(ax0, G, axis=1).astype(np.float64) / 7
                             - X.astype(np.float64)))
    assert e_rot < 0.5 * e_plain


def test_empty_and_zero_rows():
    z = np.zeros((2, 64), np.float16)
    q, a, r = oracle.quantize_rows_rotated(z, 32)
    assert np.all(q == 0) and np.all(a == 0) and np.all(r == 0)
    q, a, _ = oracle.quantize_act_groups(z, 32)
    assert np.all(q == 0) and np.all(a == 0)
    e = np.zeros((0, 64), np.float16)
    q, a, _ = oracle.quantize_rows_rotated(e, 32)
    assert q.shape == (0, 64) and a.shape == (0,)
