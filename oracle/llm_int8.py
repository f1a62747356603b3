"""CPU oracle for the LLM.int8() mixed-precision decomposition matmul Y = X.W^T.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
definition that the CUDA path is checked against. Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it; the product path
never does, and it shares no code, table or helper with the CUDA kernels.

Sources (web pages; cited by page title and section):
  [AIInfra]  Infrasys-AI/AIInfra "05Infer/06CompDistill/05Quantization01",
             LLM.int8() section: outlier detection by a magnitude threshold,
             vector-wise (row / output-column) absmax scales, INT8 matmul with
             INT32 accumulation, dequantisation by the outer product of the
             scales, FP16 matmul over the outlier dimensions, final sum.
  [Scholia]  scholia-log "Inference Quantization" notes, section 4 (scale,
             q = round(x/s), x_hat = s*q, worked INT4 example), section 5
             (outlier example), section 6 (clip to [qmin, qmax]).
  [Tanjunchen] "quantization explained part 2", section 1.2 (threshold 6.0
             on activation magnitude; per-vector INT8; the 4096-dim example
             where splitting out dim 2048 moves the scale from 70/127 to
             1/127), section 4.5 (symmetric clamp to [-qmax, qmax],
             round-half-to-even via torch.round).

Readings where the pages are silent or garbled (each also listed in the
design notes):
  * a column is an outlier iff some |x| > threshold (strict), evaluated in
    fp32 over all rows of the current X;
  * the activation absmax of a row is taken over the non-outlier columns
    only; the weight absmax of an output row over all K columns;
  * the scale factor is c = qmax/absmax (its formula is lost from the
    AIInfra page); codes are clamp(rint((x*qmax)/absmax), -qmax, qmax),
    computed as ONE fp32 product (exact: an fp16 significand times 127
    fits in 24 bits) followed by ONE correctly rounded fp32 division, and
    rint rounds half to even;
  * an all-zero row (or a row whose every column is an outlier) gets
    absmax 0 and all-zero codes;
  * outlier columns are removed from the INT8 product by zeroing their
    activation codes and keeping the full K;
  * dequantisation: C_normal = C_i32 * x_absmax * w_absmax / 127^2;
  * the FP16 outlier product and the final sum are formed in float64 and
    rounded once to fp16 (round to nearest even).

Parity status: every function below is pinned by the CPU tests (worked page
examples, closed forms, brute force on tiny inputs, error bounds, and the
threshold=inf / threshold=0 endpoints). The full-size fp16 Y has no printed
page values; it is pinned through those properties, not by page numbers.
"""
from __future__ import annotations

import numpy as np

QMAX_INT8 = 127


# ---------------------------------------------------------------------------
# Symmetric absmax quantiser ([Scholia] sections 4-6; [AIInfra] vector-wise
# quantisation; [Tanjunchen] section 4.5 for the symmetric clamp).
# ---------------------------------------------------------------------------
def absmax_codes(x: np.ndarray, absmax: np.ndarray, qmax: int) -> np.ndarray:
    """Integer codes q = clamp(rint((x*qmax)/absmax), -qmax, qmax).

    `x` is float32 (or converted to it), `absmax` broadcasts against it.
    Where absmax == 0 the code is 0 (an all-zero group has no scale to
    divide by; [Scholia] section 4 says such a tensor needs separate
    handling). Returns int32 codes.
    """
    x32 = np.asarray(x, dtype=np.float32)
    a32 = np.broadcast_to(np.asarray(absmax, dtype=np.float32), x32.shape)
    prod = x32 * np.float32(qmax)                       # exact in fp32
    safe = np.where(a32 > 0, a32, np.float32(1.0))
    with np.errstate(divide="ignore", invalid="ignore"):
        quot = prod / safe                              # one IEEE fp32 divide
    q = np.rint(quot)                                   # half to even
    q = np.clip(q, -qmax, qmax)
    q = np.where(a32 > 0, q, 0.0)
    return q.astype(np.int32)


def quantize_per_tensor(x: np.ndarray, qmax: int):
    """One scale for the whole tensor: (codes, absmax). [Scholia] section 4."""
    x32 = np.asarray(x, dtype=np.float32)
    a = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    return absmax_codes(x32, a, qmax), a


def step_size(absmax, qmax: int) -> np.ndarray:
    """Width of one integer step in real units, s = absmax/qmax ([Scholia] s4)."""
    return np.asarray(absmax, dtype=np.float64) / qmax


def dequantize_codes(q: np.ndarray, absmax, qmax: int) -> np.ndarray:
    """x_hat = s*q with s = absmax/qmax ([Scholia] section 4), in float64."""
    return np.asarray(q, dtype=np.float64) * step_size(absmax, qmax)


# ---------------------------------------------------------------------------
# Offline weight quantisation ([AIInfra] LLM.int8(): one scale per weight
# column of the h x o matrix = per output row of our [N, K] layout).
# ---------------------------------------------------------------------------
def quantize_weight_rows(W: np.ndarray):
    """W fp16 [N, K] -> (Wq int8 [N, K], w_scale fp32 [N] = row absmax over all K)."""
    W32 = np.asarray(W).astype(np.float32)
    aw = np.max(np.abs(W32), axis=1) if W32.shape[1] else np.zeros(W32.shape[0], np.float32)
    Wq = absmax_codes(W32, aw[:, None], QMAX_INT8).astype(np.int8)
    return Wq, aw.astype(np.float32)


# ---------------------------------------------------------------------------
# Outlier feature-column detection ([AIInfra] "detection: set a magnitude
# threshold", the O / not-O split; [Tanjunchen] s1.2: a channel whose
# activation magnitude exceeds the threshold, 6.0 by default).
# ---------------------------------------------------------------------------
def find_outlier_cols(X: np.ndarray, threshold: float):
    """Returns (mask bool[K], bitmap uint32[ceil(K/32)], count, idx int32 ascending).

    Column j is an outlier iff |float32(X[i, j])| > float32(threshold) for
    some row i. Bitmap bit (j % 32) of word (j // 32) is set for outliers.
    """
    X32 = np.asarray(X).astype(np.float32)
    thr = np.float32(threshold)
    K = X32.shape[1]
    mask = np.any(np.abs(X32) > thr, axis=0) if X32.shape[0] else np.zeros(K, bool)
    words = (K + 31) // 32
    bitmap = np.zeros(words, dtype=np.uint32)
    idx = np.nonzero(mask)[0].astype(np.int32)          # ascending
    for j in idx:
        bitmap[j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return mask, bitmap, int(idx.size), idx


def find_topk_cols(X: np.ndarray, k: int) -> np.ndarray:
    """Mask (bool [K]) of the k columns with the largest max |x| over the rows.

    [AIInfra] LLM.int8() section, training notes: raise the decomposition ratio
    by computing the top 1% or 2% largest-magnitude feature dimensions in FP16.
    The magnitude of a column is its max |x| over the rows (the statistic the
    threshold detection compares); ties go to the lower column index; k is
    clipped to [0, K].
    """
    X32 = np.asarray(X).astype(np.float32)
    K = X32.shape[1]
    k = max(0, min(int(k), K))
    colmax = np.max(np.abs(X32), axis=0) if X32.shape[0] else np.zeros(K, np.float32)
    order = sorted(range(K), key=lambda j: (-float(colmax[j]), j))
    mask = np.zeros(K, bool)
    mask[order[:k]] = True
    return mask


# ---------------------------------------------------------------------------
# Per-token absmax INT8 quantisation of the non-outlier part ([AIInfra]
# vector-wise quantisation of each row of X after the outliers are split
# off; [Tanjunchen] s1.2: after splitting, the remaining dims set the scale).
# ---------------------------------------------------------------------------
def quantize_act_rows(X: np.ndarray, outlier_mask: np.ndarray):
    """X fp16 [M, K] -> (Xq int8 [M, K] with 0 at outlier columns, x_scale fp32 [M])."""
    X32 = np.asarray(X).astype(np.float32)
    keep = ~np.asarray(outlier_mask, dtype=bool)
    normal = np.where(keep[None, :], np.abs(X32), np.float32(0))
    ax = np.max(normal, axis=1) if X32.shape[1] else np.zeros(X32.shape[0], np.float32)
    Xq = absmax_codes(X32, ax[:, None], QMAX_INT8)
    Xq = np.where(keep[None, :], Xq, 0).astype(np.int8)
    return Xq, ax.astype(np.float32)


# ---------------------------------------------------------------------------
# INT8 x INT8 -> INT32 matmul ([AIInfra] "C_i32 = X_i8 x W_i8", accumulated
# in INT32 to avoid overflow).
# ---------------------------------------------------------------------------
def int32_gemm(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """C[i, n] = sum_k Xq[i, k] * Wq[n, k], exact, as int32.

    Computed with a float64 library matmul: every product is an integer of
    magnitude <= 127^2 and every partial sum an integer of magnitude
    <= 127^2 * K < 2^53, so every float64 operation is exact whatever the
    library's summation order. The result must fit int32 (asserted).
    """
    A = np.asarray(Xq, dtype=np.float64)
    B = np.asarray(Wq, dtype=np.float64)
    assert 127 * 127 * A.shape[1] < 2 ** 53
    C = A @ B.T
    assert np.all(np.abs(C) <= 2 ** 31 - 1)
    return C.astype(np.int64).astype(np.int32)


def int32_dot(xq_row: np.ndarray, wq_row: np.ndarray) -> int:
    """One INT32 accumulator entry with plain Python integers."""
    return int(sum(int(a) * int(b) for a, b in zip(xq_row.tolist(), wq_row.tolist())))


# ---------------------------------------------------------------------------
# Dequantisation ([AIInfra]: C_normal ~ C_i32 / (c_x (x) c_w) with
# c = 127/absmax, i.e. C_i32 * absmax_x * absmax_w / 127^2).
# ---------------------------------------------------------------------------
def dequantize(C: np.ndarray, x_scale: np.ndarray, w_scale: np.ndarray) -> np.ndarray:
    """float64 C_normal[i, n] = C[i, n] * x_scale[i] * w_scale[n] / 127^2."""
    return (np.asarray(C, np.float64) * np.asarray(x_scale, np.float64)[:, None]
            * np.asarray(w_scale, np.float64)[None, :] / float(QMAX_INT8 * QMAX_INT8))


# ---------------------------------------------------------------------------
# FP16 outlier matmul ([AIInfra]: C_outlier = sum_{h in O} X_f16^h W_f16^h).
# ---------------------------------------------------------------------------
def outlier_gemm(X: np.ndarray, W: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """float64 C_outlier[i, n] = sum_{j in O} X[i, j] * W[n, j]."""
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size == 0:
        return np.zeros((X.shape[0], W.shape[0]), np.float64)
    return np.asarray(X, np.float64)[:, idx] @ np.asarray(W, np.float64)[:, idx].T


# ---------------------------------------------------------------------------
# Zero-point (asymmetric) per-token quantisation ([Scholia] section 6:
# q = clip(round(x/s) + z, qmin, qmax), x_hat = s(q - z), z the integer that
# represents real 0; [AIInfra] LLM.int8() section: zeropoint beats absmax below
# 6.7B because the outliers are one-sided).
# ---------------------------------------------------------------------------
ZP_QMIN, ZP_QMAX = -128, 127


def quantize_act_rows_zp(X: np.ndarray, outlier_mask: np.ndarray):
    """Per-token zero-point INT8 codes of the non-outlier columns.

    Returns (Xq int8 [M, K], step fp32 [M], zero int32 [M]). Per row, over the
    non-outlier columns: lo = min(0, min x), hi = max(0, max x) (the range keeps
    real 0 so that it maps to an integer), step = fl32(fl32(hi - lo) / 255),
    zero = clamp(-128 - rint(fl32(lo / step)), -128, 127), and
    q = clamp(rint(fl32(x / step)) + zero, -128, 127). At outlier columns q =
    zero, so (q - zero) is 0 there. A row with no nonzero kept entry gets step 0,
    zero 0 and all codes 0.
    """
    X32 = np.asarray(X).astype(np.float32)
    keep = ~np.asarray(outlier_mask, dtype=bool)
    kept = np.where(keep[None, :], X32, np.float32(0))
    hi = np.maximum(np.max(kept, axis=1), np.float32(0)) if X32.shape[1] else np.zeros(X32.shape[0], np.float32)
    lo = np.minimum(np.min(kept, axis=1), np.float32(0)) if X32.shape[1] else np.zeros(X32.shape[0], np.float32)
    step = ((hi - lo).astype(np.float32) / np.float32(255)).astype(np.float32)
    live = step > 0
    safe = np.where(live, step, np.float32(1))
    zero = np.where(live, np.clip(ZP_QMIN - np.rint((lo / safe).astype(np.float32)), ZP_QMIN, ZP_QMAX), 0)
    zero = zero.astype(np.int32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((X32 / safe[:, None]).astype(np.float32)) + zero[:, None]
    q = np.clip(q, ZP_QMIN, ZP_QMAX)
    q = np.where(live[:, None], q, 0)
    q = np.where(keep[None, :], q, zero[:, None])
    return q.astype(np.int8), step.astype(np.float32), zero


def weight_rowsum(Wq: np.ndarray) -> np.ndarray:
    """sum_k Wq[n, k] (int32 [N]), the zero-point correction's weight factor."""
    return np.sum(np.asarray(Wq, dtype=np.int64), axis=1).astype(np.int32)


def dequantize_zp(C: np.ndarray, zero: np.ndarray, step: np.ndarray, wsum: np.ndarray,
                  w_scale: np.ndarray) -> np.ndarray:
    """sum_k step*(q - zero)*w_scale/127*wq = step*w_scale/127*(C - zero*wsum), float64."""
    Ccor = (np.asarray(C, np.int64) - np.asarray(zero, np.int64)[:, None]
            * np.asarray(wsum, np.int64)[None, :])
    return (Ccor.astype(np.float64) * np.asarray(step, np.float64)[:, None]
            * np.asarray(w_scale, np.float64)[None, :] / float(QMAX_INT8))


# ---------------------------------------------------------------------------
# Full decomposition ([AIInfra]: C_f16 = C_outlier + C_normal).
# ---------------------------------------------------------------------------
def mask_to_bitmap(mask: np.ndarray):
    """(bitmap uint32[ceil(K/32)], count, idx) of a boolean column mask."""
    mask = np.asarray(mask, dtype=bool)
    K = mask.size
    bitmap = np.zeros((K + 31) // 32, dtype=np.uint32)
    idx = np.nonzero(mask)[0].astype(np.int32)
    for j in idx:
        bitmap[j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return bitmap, int(idx.size), idx


def llm_int8_matmul(X: np.ndarray, W: np.ndarray, threshold: float = 6.0,
                    Wq: np.ndarray | None = None, w_scale: np.ndarray | None = None,
                    outlier_mask: np.ndarray | None = None, zeropoint: bool = False):
    """All steps of the path; returns a dict with Y (fp16 [M, N]) and every intermediate.

    `W` is the fp16 weight [N, K]; it supplies the outlier columns of the
    FP16 product. `Wq`/`w_scale` default to quantize_weight_rows(W).
    `outlier_mask` (bool [K]) replaces the detection step with a given outlier
    set: the set of a batch whose tokens are split over several processes
    ([AIInfra]: O is a property of the batch's activations, so every part of
    the batch uses the same O); the threshold is then unused.
    `zeropoint` quantises the non-outlier part of each token with a zero point
    (quantize_act_rows_zp) instead of the symmetric absmax; x_scale then holds
    the step and the result also has `zero` and `wsum`.
    """
    X = np.asarray(X)
    W = np.asarray(W)
    if Wq is None or w_scale is None:
        Wq, w_scale = quantize_weight_rows(W)
    if outlier_mask is None:
        mask, bitmap, count, idx = find_outlier_cols(X, threshold)
    else:
        mask = np.asarray(outlier_mask, dtype=bool)
        bitmap, count, idx = mask_to_bitmap(mask)
    extra = {}
    if zeropoint:
        Xq, x_scale, zero = quantize_act_rows_zp(X, mask)
        C = int32_gemm(Xq, Wq)
        wsum = weight_rowsum(Wq)
        Cn = dequantize_zp(C, zero, x_scale, wsum, w_scale)
        extra = dict(zero=zero, wsum=wsum)
    else:
        Xq, x_scale = quantize_act_rows(X, mask)
        C = int32_gemm(Xq, Wq)
        Cn = dequantize(C, x_scale, w_scale)
    Co = outlier_gemm(X, W, idx)
    Y = (Cn + Co).astype(np.float16)
    return dict(Y=Y, mask=mask, bitmap=bitmap, count=count, idx=idx, Xq=Xq,
                x_scale=x_scale, Wq=Wq, w_scale=w_scale, C=C, C_normal=Cn, C_outlier=Co, **extra)


def llm_int8_matmul_at(X: np.ndarray, W: np.ndarray, Wq: np.ndarray, w_scale: np.ndarray,
                       threshold: float, rows: np.ndarray, cols: np.ndarray):
    """Y[rows[t], cols[t]] for sampled output positions, one by one.

    Detection runs over the whole X (the outlier set depends on every row);
    only the sampled rows are quantised and only the sampled outputs formed.
    Returns (Y_samples fp16, C_samples int32, mask, x_scale of the sampled rows).
    """
    mask, _, _, idx = find_outlier_cols(X, threshold)
    rows = np.asarray(rows, np.int64)
    cols = np.asarray(cols, np.int64)
    uniq, inv = np.unique(rows, return_inverse=True)
    Xq_r, xs_r = quantize_act_rows(np.asarray(X)[uniq], mask)
    Xq_t = Xq_r[inv].astype(np.int64)
    Wq_t = np.asarray(Wq)[cols].astype(np.int64)
    C = np.einsum("tk,tk->t", Xq_t, Wq_t)
    Cn = (C.astype(np.float64) * xs_r[inv].astype(np.float64)
          * np.asarray(w_scale, np.float64)[cols] / float(QMAX_INT8 * QMAX_INT8))
    if idx.size:
        Xo = np.asarray(X)[rows][:, idx].astype(np.float64)
        Wo = np.asarray(W)[cols][:, idx].astype(np.float64)
        Co = np.einsum("tp,tp->t", Xo, Wo)
    else:
        Co = np.zeros(rows.size, np.float64)
    return (Cn + Co).astype(np.float16), C.astype(np.int32), mask, xs_r[inv]
