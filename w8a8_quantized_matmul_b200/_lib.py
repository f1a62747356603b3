"""ctypes loader and prototypes for libint8mm.so (the C ABI in include/int8mm.h)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libint8mm.so")

I8MM_OK = 0
I8MM_ERR_INVALID_ARG = -1
I8MM_ERR_ALIGNMENT = -2
I8MM_ERR_WORKSPACE = -3
I8MM_ERR_CUDA = -4
I8MM_ERR_TIMEOUT = -5
I8MM_ERR_UNSUPPORTED_DEVICE = -6

# Every function the header declares, with its ctypes signature.
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("n_outliers", _sz), ("status", _sz), ("col_bitmap", _sz), ("col_idx", _sz),
                ("x_scale", _sz), ("Xq", _sz), ("X_O", _sz), ("W_O", _sz), ("total", _sz),
                ("panel_ld", _i)]


PROTOTYPES = {
    "int8_quantize_weight_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "int8_transpose_weight": (_i, [_vp, _i, _i, _vp, _vp]),
    "int8_find_outlier_cols": (_i, [_vp, _i, _i, _f, _vp, _vp, _vp, _vp]),
    "int8_quantize_act_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp]),
    "int8_mixed_matmul_workspace_size": (_sz, [_i, _i, _i]),
    "int8_mixed_matmul_workspace_layout": (_i, [_i, _i, _i, ctypes.POINTER(WorkspaceLayout)]),
    "int8_mixed_matmul": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "int8_mixed_matmul_profiled": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp, _vp, _sz, _vp,
                                        ctypes.POINTER(_vp)]),
    "int8_mixed_matmul_stage": (_i, [_i, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "int8_mixed_matmul_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp, _vp]),
    "int8_mixed_matmul_sharded": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _i, _vp, _vp, _sz,
                                       _vp]),
    "int8_debug_gemm_i32": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp]),
    "int8_column_absmax": (_i, [_vp, _i, _i, _vp, _vp]),
    "int8_weight_rowsum": (_i, [_vp, _i, _i, _vp, _vp]),
    "int8_mixed_matmul_zp_workspace_size": (_sz, [_i, _i, _i]),
    "int8_mixed_matmul_zp": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "int8_mixed_matmul_topk_workspace_size": (_sz, [_i, _i, _i]),
    "int8_mixed_matmul_topk": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "int8_smoothquant_factors": (_i, [_vp, _vp, _i, _f, _vp, _vp, _vp]),
    "int8_smoothquant_weight_rows": (_i, [_vp, _vp, _i, _i, _vp, _vp, _vp]),
    "int8_smoothquant_workspace_size": (_sz, [_i, _i, _i]),
    "int8_smoothquant_matmul": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "int8_rotate_quantize_rows": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "int8_rotated_workspace_size": (_sz, [_i, _i, _i]),
    "int8_rotated_matmul": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "int4_rotate_quantize_groups": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "int4_rotate_quantize_weight_blocks": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "int4_unpack": (_i, [_vp, _i, _i, _vp, _vp]),
    "int4_rotated_workspace_size": (_sz, [_i, _i, _i, _i]),
    "int4_rotated_matmul": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "int8_selftest_wait_timeout": (_i, [_vp, _vp]),
    "int8_device_status": (_i, [_vp, _vp]),
    "int8_noalloc_device_status": (_i, [_vp]),
    "int8_status_string": (ctypes.c_char_p, [_i]),
    "int8_last_error_string": (ctypes.c_char_p, []),
}

_lib = None


class Int8mmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = ""
        if status == I8MM_ERR_CUDA:
            detail = ": " + load().int8_last_error_string().decode()
        super().__init__(f"{fn} failed: {status} ({status_string(status)}){detail}")


def load() -> ctypes.CDLL:
    """Loads the in-tree library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m w8a8_quantized_matmul_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().int8_status_string(status).decode()


def check(fn: str, status: int) -> None:
    if status != I8MM_OK:
        raise Int8mmError(fn, status)
