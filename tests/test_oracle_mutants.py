"""Planted mistakes in a copy of the oracle must each fail a pin.

Each mutant rewrites one line of a temporary copy of oracle/llm_int8.py
(a dropped term, a wrong comparison, a wrong rounding mode, a transposed
or reversed operand, a wrong sign) and runs tests/test_oracle_pins.py
against it in a subprocess. Nothing here touches a GPU.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "dequant_over_127_not_127sq": ("/ float(QMAX_INT8 * QMAX_INT8))\n\n\n#", "/ float(QMAX_INT8))\n\n\n#"),
    "detect_ge_not_gt": ("np.abs(X32) > thr", "np.abs(X32) >= thr"),
    "round_half_up": ("q = np.rint(quot)", "q = np.floor(quot + 0.5)"),
    "gemm_reversed_k": ("C = A @ B.T", "C = A @ B[:, ::-1].T"),
    "act_absmax_over_all_cols": ("normal = np.where(keep[None, :], np.abs(X32), np.float32(0))",
                                 "normal = np.abs(X32)"),
    "outlier_sign_flipped": ("return np.asarray(X, np.float64)[:, idx] @",
                             "return -np.asarray(X, np.float64)[:, idx] @"),
    "outlier_term_dropped": ("Y = (Cn + Co).astype(np.float16)", "Y = (Cn).astype(np.float16)"),
    "w_scale_index_reversed": ("* np.asarray(w_scale, np.float64)[None, :] /",
                               "* np.asarray(w_scale, np.float64)[::-1][None, :] /"),
    "weight_absmax_per_tensor": ("aw = np.max(np.abs(W32), axis=1)",
                                 "aw = np.max(np.abs(W32), axis=1) * 0 + np.max(np.abs(W32))"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "llm_int8.py")).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation site for {name} no longer exists"
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "llm_int8.py").write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
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


TOPK_MUTANTS = {
    "topk_ties_to_higher_index": ("key=lambda j: (-float(colmax[j]), j))", "key=lambda j: (-float(colmax[j]), -j))"),
    "topk_one_extra_column": ("mask[order[:k]] = True", "mask[order[:k + 1]] = True"),
    "topk_by_mean_magnitude": ("colmax = np.max(np.abs(X32), axis=0) if X32.shape[0] else np.zeros(K, np.float32)\n    order",
                               "colmax = np.mean(np.abs(X32), axis=0) if X32.shape[0] else np.zeros(K, np.float32)\n    order"),
}


@pytest.mark.parametrize("name", sorted(TOPK_MUTANTS))
def test_topk_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "llm_int8.py")).read()
    old, new = TOPK_MUTANTS[name]
    assert old in src, f"mutation site for {name} no longer exists"
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "llm_int8.py").write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_topk_pins.py"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


ZP_MUTANTS = {
    "zp_zero_sign_flipped": ("zero = np.where(live, np.clip(ZP_QMIN - np.rint((lo / safe).astype(np.float32)), ZP_QMIN, ZP_QMAX), 0)",
                             "zero = np.where(live, np.clip(ZP_QMIN + np.rint((lo / safe).astype(np.float32)), ZP_QMIN, ZP_QMAX), 0)"),
    "zp_range_without_zero": ("lo = np.minimum(np.min(kept, axis=1), np.float32(0))",
                              "lo = np.min(np.where(keep[None, :], X32, np.float32(np.inf)), axis=1) + 0 * np.float32(0)"),
    "zp_correction_dropped": ("Ccor = (np.asarray(C, np.int64) - np.asarray(zero, np.int64)[:, None]",
                              "Ccor = (np.asarray(C, np.int64) - 0 * np.asarray(zero, np.int64)[:, None]"),
    "zp_step_over_127": ("step = ((hi - lo).astype(np.float32) / np.float32(255)).astype(np.float32)",
                         "step = ((hi - lo).astype(np.float32) / np.float32(127)).astype(np.float32)"),
}


@pytest.mark.parametrize("name", sorted(ZP_MUTANTS))
def test_zeropoint_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "llm_int8.py")).read()
    old, new = ZP_MUTANTS[name]
    assert old in src, f"mutation site for {name} no longer exists"
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "llm_int8.py").write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_zeropoint_pins.py"], cwd=tmp_path, capture_output=True,
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
