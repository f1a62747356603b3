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
    int32_dot,
    dequantize,
    outlier_gemm,
    llm_int8_matmul,
    llm_int8_matmul_at,
)
from .llm_int8 import (  # noqa: F401,E402
    mask_to_bitmap, find_topk_cols, quantize_act_rows_zp, weight_rowsum, dequantize_zp,
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
