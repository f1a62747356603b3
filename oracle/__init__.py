"""CPU oracle (test infrastructure only; see llm_int8.py)."""
from .llm_int8 import (  # noqa: F401
    QMAX_INT8,
    absmax_codes,
    quantize_per_tensor,
    step_size,
    dequantize_codes,
    quantize_weight_rows,
    find_outlier_cols,
    quantize_act_rows,
    int32_gemm,
    dequantize,
    outlier_gemm,
    llm_int8_matmul,
    llm_int8_matmul_at,
)
from .llm_int8 import (  # noqa: F401,E402
    mask_to_bitmap, find_topk_cols, quantize_act_rows_zp, weight_rowsum, dequantize_zp,
    half_to_float, double_to_half, threads, set_threads, lib,
    ZP_QMIN, ZP_QMAX,
)
from .smoothquant import (  # noqa: F401,E402
    column_absmax,
    smooth_factors,
    smooth_weight_rows,
    smooth_rcp,
    smooth_act_rows,
    smoothquant_matmul,
    per_tensor_quant_dequant,
)
from .rotation import (  # noqa: F401,E402
    QMAX_W8,
    QMAX_W4,
    hadamard,
    rotation_scale,
    hadamard_sums,
    rotate_groups,
    rotate_groups_f64,
    quantize_rows_rotated,
    rotated_w8a8_matmul,
    quantize_act_groups,
    quantize_weight_blocks,
    pack_int4,
    unpack_int4,
    group_gemm,
    dequantize_groups,
    rotated_w4a4_matmul,
)
