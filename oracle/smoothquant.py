"""CPU oracle for the SmoothQuant W8A8 matmul (TEST INFRASTRUCTURE ONLY).

The plain, slow definition the CUDA SmoothQuant path is checked against. Only
the tests, the smoke check and the benchmark's CPU-baseline leg may use it; it
shares no code with the CUDA kernels.

Source: [Tanjunchen] "quantization explained part 2", section 4 (SmoothQuant):
  4.2  Y = X.W = (X diag(s)^-1)(diag(s) W) = X_hat . W_hat: per input channel
       i the activations are divided by s_i and the weights multiplied by s_i,
       which leaves the product unchanged; s_i = max|X_i|^alpha /
       max|W_i|^(1-alpha) with the migration strength alpha (typically 0.5).
  4.2  after the migration the activations quantise well, so both operands
       are INT8 and the product runs on the INT8 tensor cores (W8A8).
  4.4  the factors are computed offline (from calibration activations).
  4.5  a toy example: 16 channels, 32 tokens, one channel x60, per-tensor
       INT8 quantise-dequantise of both operands; the mean |error| of the
       output falls from 0.108 to 0.054 with alpha = 0.5.

Readings (each also in the design notes):
  * W is stored [N][K] (out x in), so "max|W_i|" for input channel i is the
    max over the N output rows of column i, and diag(s) W multiplies column
    i of our W by s_i;
  * a channel with max|X_i| = 0 or max|W_i| = 0 gets s_i = 1 (nothing to
    migrate; the formula would divide by zero or give 0);
  * s is an offline fp32 vector; the runtime multiplies X by r = fl32(1/s)
    (X_hat = fl32(x * r_i)), and the weight side by s (W_hat = fl32(w * s_i));
  * the INT8 scheme after smoothing is the vector-wise one of the LLM.int8()
    path here (per token for X_hat, per output row for W_hat, codes
    clamp(rint(fl32(x*127)/absmax), +-127)); the page's toy example uses one
    scale per tensor, which `per_tensor_quant_dequant` reproduces for its pin;
  * no outlier split: every column goes through the INT8 product;
  * dequantisation and output as in the LLM.int8() path: C * x_absmax *
    w_absmax / 127^2 in float64, rounded once to fp16.

Parity status: the factors, the smoothing, the quantisers and the product are
pinned by the CPU tests (the section 4.5 example's printed errors, the exact
equivalence X_hat.W_hat = X.W, closed forms for alpha = 0, 0.5 and 1, brute
force on tiny inputs).
"""
from __future__ import annotations

import numpy as np

from .llm_int8 import QMAX_INT8, absmax_codes, int32_gemm


def column_absmax(X: np.ndarray) -> np.ndarray:
    """max over rows of |X[:, i]| for each column i, fp32 [K] (calibration statistic)."""
    X32 = np.asarray(X).astype(np.float32)
    if X32.shape[0] == 0:
        return np.zeros(X32.shape[1], np.float32)
    return np.max(np.abs(X32), axis=0)


def smooth_factors(act_absmax: np.ndarray, W: np.ndarray, alpha: float) -> np.ndarray:
    """s_i = act_absmax_i^alpha / max_n|W[n, i]|^(1 - alpha), float64 [K]; 1 where either is 0."""
    a = np.asarray(act_absmax, dtype=np.float64)
    w = np.max(np.abs(np.asarray(W).astype(np.float64)), axis=0)
    ok = (a > 0) & (w > 0)
    s = np.ones_like(a)
    s[ok] = a[ok] ** alpha / w[ok] ** (1.0 - alpha)
    return s


def smooth_weight_rows(W: np.ndarray, s32: np.ndarray):
    """W_hat = fl32(W * s) per input column, quantised per output row.

    Returns (Wq int8 [N, K], w_scale fp32 [N] = row absmax of W_hat, W_hat fp32)."""
    s32 = np.asarray(s32, dtype=np.float32)
    W_hat = np.asarray(W).astype(np.float32) * s32[None, :]
    aw = (np.max(np.abs(W_hat), axis=1) if W_hat.shape[1]
          else np.zeros(W_hat.shape[0], np.float32))
    Wq = absmax_codes(W_hat, aw[:, None], QMAX_INT8).astype(np.int8)
    return Wq, aw.astype(np.float32), W_hat


def smooth_rcp(s32: np.ndarray) -> np.ndarray:
    """r = fl32(1 / s), the runtime multiplier of X."""
    return (np.float32(1.0) / np.asarray(s32, dtype=np.float32)).astype(np.float32)


def smooth_act_rows(X: np.ndarray, r32: np.ndarray):
    """X_hat = fl32(x * r) per column; per-token absmax INT8 codes.

    Returns (Xq int8 [M, K], x_scale fp32 [M] = row absmax of X_hat, X_hat fp32)."""
    X_hat = np.asarray(X).astype(np.float32) * np.asarray(r32, dtype=np.float32)[None, :]
    ax = (np.max(np.abs(X_hat), axis=1) if X_hat.shape[1]
          else np.zeros(X_hat.shape[0], np.float32))
    Xq = absmax_codes(X_hat, ax[:, None], QMAX_INT8).astype(np.int8)
    return Xq, ax.astype(np.float32), X_hat


def smoothquant_matmul(X: np.ndarray, Wq: np.ndarray, w_scale: np.ndarray, r32: np.ndarray):
    """The runtime W8A8 path: smooth and quantise X, INT8 product, dequantise.

    Returns a dict with Y (fp16 [M, N]), Xq, x_scale, X_hat and C (int32)."""
    Xq, x_scale, X_hat = smooth_act_rows(X, r32)
    C = int32_gemm(Xq, Wq)
    Y64 = (np.asarray(C, np.float64) * np.asarray(x_scale, np.float64)[:, None]
           * np.asarray(w_scale, np.float64)[None, :] / float(QMAX_INT8 * QMAX_INT8))
    return dict(Y=Y64.astype(np.float16), Xq=Xq, x_scale=x_scale, X_hat=X_hat, C=C)


def per_tensor_quant_dequant(x: np.ndarray, qmax: int = QMAX_INT8) -> np.ndarray:
    """One step s = max|x|/qmax for the whole tensor; s * clamp(rint(x/s)), float64
    (the quantise-dequantise of the section 4.5 example)."""
    x = np.asarray(x, dtype=np.float64)
    step = np.max(np.abs(x)) / qmax
    if step == 0:
        return np.zeros_like(x)
    return np.clip(np.rint(x / step), -qmax, qmax) * step
