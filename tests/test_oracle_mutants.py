"""Planted mistakes in a copy of the oracle must each fail a pin.

Each mutant rewrites one line of a temporary copy of an oracle source (a
dropped term, a wrong comparison, a wrong rounding mode, a transposed or
reversed operand, a wrong sign, a missing check): the C++ oracle
(oracle/llm_int8.cpp, rebuilt into a temporary library that the shim loads
through LLM_INT8_ORACLE_LIB) or one of the numpy oracles of the other rows.
The pins of the changed part then run in a subprocess and must fail. Nothing
here touches a GPU.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Each entry: (text in oracle/llm_int8.cpp, its planted replacement, pins file).
CPP_MUTANTS = {
    "dequant_over_127_not_127sq": ("static_cast<double>(ws[n]) / 16129.0;",
                                   "static_cast<double>(ws[n]) / 127.0;", "test_oracle_pins.py"),
    "detect_ge_not_gt": ("* K + j])) > threshold) out = true;",
                         "* K + j])) >= threshold) out = true;", "test_oracle_pins.py"),
    "round_half_up": ("const float q = std::rint(quot);", "const float q = std::floor(quot + 0.5f);",
                      "test_oracle_pins.py"),
    "gemm_reversed_k": ("s += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);",
                        "s += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[K - 1 - k]);",
                        "test_oracle_pins.py"),
    "act_absmax_over_all_cols": ("if (!mask[j]) a = std::max(a, std::fabs(half_to_float(x[j])));",
                                 "a = std::max(a, std::fabs(half_to_float(x[j])));",
                                 "test_oracle_pins.py"),
    "outlier_sign_flipped": ("        s += half_to_double(X[i * K + idx[p]])",
                             "        s -= half_to_double(X[i * K + idx[p]])", "test_oracle_pins.py"),
    "outlier_term_dropped": ("Y[e] = double_to_half(Cn[e] + Co[e]);", "Y[e] = double_to_half(Cn[e]);",
                             "test_oracle_pins.py"),
    "w_scale_index_reversed": ("static_cast<double>(ws[n]) / 16129.0;",
                               "static_cast<double>(ws[N - 1 - n]) / 16129.0;", "test_oracle_pins.py"),
    "weight_absmax_over_half_the_row": (
        "for (int k = 0; k < K; ++k) a = std::max(a, std::fabs(half_to_float(w[k])));",
        "for (int k = 0; k < K / 2; ++k) a = std::max(a, std::fabs(half_to_float(w[k])));",
        "test_oracle_pins.py"),
    "half_decode_exponent_bias": ("static_cast<float>(1024 + f), e - 25);",
                                  "static_cast<float>(1024 + f), e - 24);", "test_oracle_pins.py"),
    "half_encode_ties_away": ("double q = std::nearbyint(std::ldexp(a, 10 - E));",
                              "double q = std::round(std::ldexp(a, 10 - E));", "test_oracle_pins.py"),
    "half_decode_subnormal_scale": ("v = std::ldexp(static_cast<float>(f), -24);",
                                    "v = std::ldexp(static_cast<float>(f), -25);", "test_oracle_pins.py"),
    "gemm_overflow_unchecked": ("if (s > INT32_MAX || s < INT32_MIN) bad[i] = 1;", "",
                                "test_oracle_pins.py"),
    "topk_ties_to_higher_index": ("[&](int p, int q) { return colmax[p] > colmax[q]; });",
                                  "[&](int p, int q) { return colmax[p] > colmax[q] || "
                                  "(colmax[p] == colmax[q] && p > q); });", "test_topk_pins.py"),
    "topk_one_extra_column": ("for (int t = 0; t < k; ++t) mask[order[t]] = 1;",
                              "for (int t = 0; t < k + 1 && t < K; ++t) mask[order[t]] = 1;",
                              "test_topk_pins.py"),
    "topk_by_mean_magnitude": ("colmax[j] = std::max(colmax[j], std::fabs(",
                               "colmax[j] = colmax[j] + (std::fabs(", "test_topk_pins.py"),
    "zp_zero_sign_flipped": ("-128.0f - std::rint(lq)", "-128.0f + std::rint(lq)",
                             "test_zeropoint_pins.py"),
    "zp_range_without_zero": ("float lo = 0.0f, hi = 0.0f;", "float lo = INFINITY, hi = 0.0f;",
                              "test_zeropoint_pins.py"),
    "zp_correction_dropped": ("static_cast<int64_t>(zero[i]) * static_cast<int64_t>(wsum[n]);",
                              "0 * static_cast<int64_t>(wsum[n]);", "test_zeropoint_pins.py"),
    "zp_step_over_127": ("const float step = range / 255.0f;", "const float step = range / 127.0f;",
                         "test_zeropoint_pins.py"),
}


@pytest.mark.parametrize("name", sorted(CPP_MUTANTS))
def test_pins_catch_planted_mistake_in_cpp_oracle(name, tmp_path):
    sys.path.insert(0, ROOT)
    from oracle import build as obuild
    src = open(os.path.join(ROOT, "oracle", "llm_int8.cpp")).read()
    old, new, pins = CPP_MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} no longer exists"
    mutant = tmp_path / "llm_int8.cpp"
    mutant.write_text(src.replace(old, new, 1))
    so = obuild.build(str(mutant), str(tmp_path / "liborc_mutant.so"), force=True)
    env = dict(os.environ, LLM_INT8_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join("tests", pins)], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


SQ_MUTANTS = {
    "sq_x_multiplied_by_s": ("return (np.float32(1.0) / np.asarray(s32, dtype=np.float32)).astype(np.float32)",
                             "return np.asarray(s32, dtype=np.float32).copy()"),
    "sq_alpha_swapped": ("s[ok] = a[ok] ** alpha / w[ok] ** (1.0 - alpha)",
                         "s[ok] = a[ok] ** (1.0 - alpha) / w[ok] ** alpha"),
    "sq_weight_not_scaled": ("W_hat = np.asarray(W).astype(np.float32) * s32[None, :]",
                             "W_hat = np.asarray(W).astype(np.float32)"),
    "sq_dequant_over_127": ("* np.asarray(w_scale, np.float64)[None, :] / float(QMAX_INT8 * QMAX_INT8))",
                            "* np.asarray(w_scale, np.float64)[None, :] / float(QMAX_INT8))"),
    "sq_weight_max_over_rows": ("w = np.max(np.abs(np.asarray(W).astype(np.float64)), axis=0)",
                                "w = np.max(np.abs(np.asarray(W).astype(np.float64))) + 0 * np.asarray(act_absmax)"),
}


@pytest.mark.parametrize("name", sorted(SQ_MUTANTS))
def test_smoothquant_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "smoothquant.py")).read()
    old, new = SQ_MUTANTS[name]
    assert old in src, f"mutation site for {name} no longer exists"
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "smoothquant.py").write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_smoothquant_pins.py"], cwd=tmp_path, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


ROT_MUTANTS = {
    "rot_normalised_by_g": ("return np.float32(1.0 / np.sqrt(float(G)))",
                            "return np.float32(1.0 / float(G))"),
    "rot_f64_normalised_by_g": ("return hadamard_sums(X, G) / np.sqrt(float(G))",
                                "return hadamard_sums(X, G) / float(G)"),
    "rot_sylvester_sign_moved": ("H = np.block([[H, H], [H, -H]])",
                                 "H = np.block([[H, -H], [H, H]])"),
    "rot_matrix_rows_reversed": ("S[:, g * G:(g + 1) * G] = Xf[:, g * G:(g + 1) * G] @ H",
                                 "S[:, g * G:(g + 1) * G] = Xf[:, g * G:(g + 1) * G] @ H[::-1]"),
    "rot_scaled_before_rounding": ("return S.astype(np.float32) * rotation_scale(G)",
                                   "return (S * float(rotation_scale(G))).astype(np.float32)"),
    "w4_block_absmax_first_row_only": ("a = np.abs(r).reshape(N // G, G, K // G, G).max(axis=(1, 3))",
                                       "a = np.abs(r).reshape(N // G, G, K // G, G)[:, :1].max(axis=(1, 3))"),
    "w4_pack_nibbles_reversed": ("return np.bitwise_or.reduce(nib << shifts, axis=2).astype(np.uint32)",
                                 "return np.bitwise_or.reduce(nib << shifts[:, :, ::-1], axis=2).astype(np.uint32)"),
    "w4_dequant_block_index_tiled": ("awn = np.repeat(np.asarray(aw, np.float64), G, axis=0)",
                                     "awn = np.tile(np.asarray(aw, np.float64), (G, 1))"),
    "w8_rot_dequant_over_127": ("/ float(QMAX_W8 * QMAX_W8))", "/ float(QMAX_W8))"),
    "w4_act_absmax_over_whole_row": (
        "a = np.abs(r).reshape(rows, K // G, G).max(axis=2) if K",
        "a = np.abs(r).reshape(rows, K // G, G).max(axis=(1, 2))[:, None] * np.ones((1, K // G), np.float32) if K"),
}


@pytest.mark.parametrize("name", sorted(ROT_MUTANTS))
def test_rotation_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "rotation.py")).read()
    old, new = ROT_MUTANTS[name]
    assert old in src, f"mutation site for {name} no longer exists"
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "rotation.py").write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_rotation_pins.py"], cwd=tmp_path, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
