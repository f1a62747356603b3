"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

* the library builds for sm_100a and exports every function include/int8mm.h declares;
* argument validation returns the documented status before any launch;
* the workspace layout is aligned, non-overlapping and matches the size query.
"""
import ctypes
import math
import os
import re

import pytest

from w8a8_quantized_matmul_b200 import _lib
from w8a8_quantized_matmul_b200 import build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int8mm.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(int[48]_[a-z0-9_]+)\s*\(", src, re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["int8_quantize_weight_rows", "int8_find_outlier_cols", "int8_quantize_act_rows",
                     "int8_mixed_matmul", "int8_mixed_matmul_workspace_size", "int8_debug_gemm_i32",
                     "int8_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in int8mm.h but not exported"
        assert name in _lib.PROTOTYPES, f"{name} has no ctypes prototype"


def test_library_is_built_for_sm100a(lib):
    # The fatbinary embeds the target architecture name.
    blob = open(_lib.LIB_PATH, "rb").read()
    assert b"sm_100a" in blob


def test_status_strings(lib):
    for code in range(-6, 1):
        assert lib.int8_status_string(code)
    assert b"unknown" in lib.int8_status_string(42)


# Fake, 256-byte aligned "device" addresses: validation must reject the call
# before anything dereferences or launches, so these are never touched.
A = 1 << 20
A2 = 2 << 20
MIS = A + 8


def _mm(lib, X=A, Wq=A, ws=A, W=A, M=64, N=64, K=64, thr=6.0, Y=A, wsp=A, wsb=None):
    if wsb is None:
        wsb = lib.int8_mixed_matmul_workspace_size(M, N, K) if M >= 0 and N >= 0 else 0
    return lib.int8_mixed_matmul(X, Wq, ws, W, M, N, K, thr, Y, wsp, wsb, None)


def test_mixed_matmul_validation(lib):
    assert _mm(lib, K=0) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, K=24) == _lib.I8MM_ERR_ALIGNMENT
    assert _mm(lib, K=-16) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, M=-1) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, N=-1) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, K=65536 + 16) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, thr=math.nan) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, thr=-1.0) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, X=None) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, Wq=None) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, ws=None) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, W=None) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, Y=None) == _lib.I8MM_ERR_INVALID_ARG
    assert _mm(lib, X=MIS) == _lib.I8MM_ERR_ALIGNMENT
    assert _mm(lib, Y=MIS) == _lib.I8MM_ERR_ALIGNMENT
    assert _mm(lib, W=MIS) == _lib.I8MM_ERR_ALIGNMENT
    assert _mm(lib, wsp=None) == _lib.I8MM_ERR_WORKSPACE
    need = lib.int8_mixed_matmul_workspace_size(64, 64, 64)
    assert _mm(lib, wsb=need - 1) == _lib.I8MM_ERR_WORKSPACE
    assert _mm(lib, wsp=A + 16) == _lib.I8MM_ERR_ALIGNMENT
    # Empty problems are valid and launch nothing.
    assert _mm(lib, M=0) == _lib.I8MM_OK
    assert _mm(lib, N=0) == _lib.I8MM_OK
    assert _mm(lib, M=0, X=None, Y=None, wsp=None, wsb=0) == _lib.I8MM_OK


def test_other_entry_points_validation(lib):
    assert lib.int8_quantize_weight_rows(A, 8, 40, A, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_quantize_weight_rows(None, 8, 64, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_quantize_weight_rows(A, 8, 64, MIS, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_quantize_weight_rows(A, 0, 64, None, None, None) == _lib.I8MM_OK
    assert lib.int8_transpose_weight(A, 8, 40, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_transpose_weight(None, 8, 64, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_transpose_weight(A, 8, 64, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_transpose_weight(A, 8, 64, MIS, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_transpose_weight(A, -1, 64, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_transpose_weight(A, 0, 64, None, None) == _lib.I8MM_OK
    assert lib.int8_find_outlier_cols(A, 4, 64, math.nan, A, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_find_outlier_cols(A, 4, 64, -0.5, A, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_find_outlier_cols(A, 4, 64, 6.0, None, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_find_outlier_cols(None, 4, 64, 6.0, A, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_find_outlier_cols(A, 4, 64, 6.0, A, None, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_find_outlier_cols(A, 4, 64, 6.0, A, A, MIS, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_find_outlier_cols(A, 4, 8, 6.0, A, A, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_quantize_act_rows(A, 4, 64, None, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_quantize_act_rows(A, 4, 64, A, MIS, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_quantize_act_rows(A, 0, 64, None, None, None, None) == _lib.I8MM_OK
    assert lib.int8_debug_gemm_i32(A, A, 4, 4, 20, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_debug_gemm_i32(A, None, 4, 4, 32, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_debug_gemm_i32(A, A, 0, 4, 32, A, None) == _lib.I8MM_OK
    assert lib.int8_device_status(None, None) == _lib.I8MM_ERR_INVALID_ARG
    need = lib.int8_mixed_matmul_workspace_size(64, 64, 64)
    assert lib.int8_mixed_matmul_stage(3, A, A, A, A, 64, 64, 64, 6.0, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_mixed_matmul_stage(1, A, A, A, A, 64, 64, 24, 6.0, A, A, need, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_mixed_matmul_stage(2, A, A, A, A, 64, 64, 64, 6.0, A, None, need, None) == _lib.I8MM_ERR_WORKSPACE
    ev = (ctypes.c_void_p * 3)(None, None, None)
    assert lib.int8_mixed_matmul_profiled(A, A, A, A, 64, 64, 64, 6.0, A, A, need, None, ev) == _lib.I8MM_ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (16, 256, 256), (200, 264, 272), (2048, 16384, 4096),
                                   (4096, 28672, 8192), (17, 8, 48)])
def test_workspace_layout(lib, M, N, K):
    lay = _lib.WorkspaceLayout()
    assert lib.int8_mixed_matmul_workspace_layout(M, N, K, ctypes.byref(lay)) == _lib.I8MM_OK
    assert lay.total == lib.int8_mixed_matmul_workspace_size(M, N, K)
    assert lay.panel_ld % 64 == 0 and lay.panel_ld >= K and lay.panel_ld - K < 64
    words = (K + 31) // 32
    regions = [(lay.n_outliers, 4), (lay.status, 4), (lay.col_bitmap, 4 * words), (lay.col_idx, 4 * K),
               (lay.x_scale, 4 * M), (lay.Xq, M * K), (lay.X_O, 2 * M * lay.panel_ld),
               (lay.W_O, 2 * N * lay.panel_ld)]
    for off, size in regions:
        assert off % 4 == 0 and off + size <= lay.total
    for off, _ in regions[2:]:
        assert off % 16 == 0
    for off in (lay.Xq, lay.X_O, lay.W_O, lay.x_scale, lay.col_idx):
        assert off % 256 == 0
    spans = sorted(regions)
    for (o1, s1), (o2, _) in zip(spans, spans[1:]):
        assert o1 + s1 <= o2, "workspace regions overlap"


def test_workspace_size_rejects_bad_sizes(lib):
    assert lib.int8_mixed_matmul_workspace_size(4, 4, 20) == 0
    assert lib.int8_mixed_matmul_workspace_size(-1, 4, 32) == 0
    lay = _lib.WorkspaceLayout()
    assert lib.int8_mixed_matmul_workspace_layout(4, 4, 20, ctypes.byref(lay)) == _lib.I8MM_ERR_ALIGNMENT


def test_rotation_entry_points_validation(lib):
    # G must be a power of two in [16, 256] dividing K; K <= 32768
    assert lib.int8_rotate_quantize_rows(A, 4, 256, 24, A, A, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotate_quantize_rows(A, 4, 256, 512, A, A, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotate_quantize_rows(A, 4, 96, 64, A, A, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotate_quantize_rows(A, 4, 65536, 128, A, A, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotate_quantize_rows(None, 4, 256, 128, A, A, None, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotate_quantize_rows(A, 4, 256, 128, MIS, A, None, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_rotate_quantize_rows(A, 4, 256, 128, A, A, MIS, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_rotate_quantize_rows(A, 0, 256, 128, None, None, None, None) == _lib.I8MM_OK
    need = lib.int8_rotated_workspace_size(64, 64, 256)
    assert need > 64 * 256
    assert lib.int8_rotated_workspace_size(64, 64, 65536) == 0
    assert lib.int8_rotated_matmul(A, A, A, 64, 64, 256, 128, A, A, need - 1, None) == _lib.I8MM_ERR_WORKSPACE
    assert lib.int8_rotated_matmul(A, A, A, 64, 64, 256, 48, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int8_rotated_matmul(A, A, A, 64, 64, 256, 128, MIS, A, need, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_rotated_matmul(A, A, A, 64, 64, 256, 128, A, A + 16, need, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int8_rotated_matmul(A, A, A, 0, 64, 256, 128, A, None, 0, None) == _lib.I8MM_OK
    assert lib.int4_rotate_quantize_groups(A, 4, 256, 128, None, None, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotate_quantize_groups(A, 4, 256, 128, A, A + 4, A, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int4_rotate_quantize_groups(A, 4, 256, 8, A, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotate_quantize_weight_blocks(A, 96, 256, 64, A, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotate_quantize_weight_blocks(A, 128, 256, 64, None, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotate_quantize_weight_blocks(A, 0, 256, 64, None, None, None) == _lib.I8MM_OK


def test_int4_entry_points_validation(lib):
    # unpack: K % 32, 16-byte alignment, empty
    assert lib.int4_unpack(A, 4, 48, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_unpack(A, 4, 64, MIS, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int4_unpack(None, 4, 64, A, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_unpack(None, 0, 64, None, None) == _lib.I8MM_OK
    # W4A4 matmul: G in {64, 128, 256}, K % 128, N % G, workspace
    need = lib.int4_rotated_workspace_size(64, 256, 512, 128)
    assert need >= 64 * 512 + 4 * 64 * 4
    assert lib.int4_rotated_workspace_size(64, 256, 520, 128) == 0
    assert lib.int4_rotated_matmul(A, A, A, 64, 256, 512, 32, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotated_matmul(A, A, A, 64, 256, 320, 64, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotated_matmul(A, A, A, 64, 200, 512, 128, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotated_matmul(A, A, A, 64, 256, 512, 128, A, A, need - 1, None) == _lib.I8MM_ERR_WORKSPACE
    assert lib.int4_rotated_matmul(A, A, A, 64, 256, 512, 128, A, A + 16, need, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int4_rotated_matmul(MIS, A, A, 64, 256, 512, 128, A, A, need, None) == _lib.I8MM_ERR_ALIGNMENT
    assert lib.int4_rotated_matmul(A, None, A, 64, 256, 512, 128, A, A, need, None) == _lib.I8MM_ERR_INVALID_ARG
    assert lib.int4_rotated_matmul(A, A, A, 0, 256, 512, 128, A, None, 0, None) == _lib.I8MM_OK
    # self-test hook: a status pointer is required
    assert lib.int8_selftest_wait_timeout(None, None) == _lib.I8MM_ERR_INVALID_ARG


def test_header_is_plain_c(tmp_path):
    """include/int8mm.h compiles as C99 (pedantic) and as C++17 on its own."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    src = tmp_path / "use_header.c"
    src.write_text('#include "int8mm.h"\nint main(void) { return I8MM_OK; }\n')
    inc = os.path.join(ROOT, "include")
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, "-c",
                 str(src), "-o", str(tmp_path / "a.o")],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", inc, "-x", "c++", "-c",
                 str(src), "-o", str(tmp_path / "b.o")]):
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_plain_c_program_links_and_calls_the_library(lib, tmp_path):
    """A C program (tests/c_consumer.c) links libint8mm.so through the header
    and exercises the entry points that need no GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "c_consumer"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_consumer.c"), "-L", libdir, "-lint8mm",
                        "-Wl,-rpath," + libdir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr + r.stdout
    assert "c consumer ok" in r.stdout
