"""CPU oracle for grouped Hadamard rotation before quantisation (TEST INFRASTRUCTURE ONLY).

The plain, slow definition the CUDA rotation path is checked against. Only the
tests, the smoke check and the benchmark's CPU-baseline leg may use it; it
shares no code with the CUDA kernels.

Source: [Baidu] developer.baidu.com article "低比特量化加速：分组旋转方法从W8A8到
W4A4的实践与展望" (grouped rotation from W8A8 to W4A4):
  section 2   before quantising, apply an invertible orthogonal transform so
              that the values suit low-bit codes; apply it per group
              (sub-block) rather than to the whole matrix; the transform is a
              regular (normalised) Hadamard matrix: fixed entries, orthogonal,
              cheap; no training and no calibration data are needed;
  section 3   W8A8 = 8-bit weights and activations; W4A4 = 4-bit, 16 levels;
  section 5.1 the weight is cut into G x G sub-blocks, each multiplied by the
              normalised Hadamard matrix, quantisation parameters are taken
              per sub-block, and the 4-bit integers are packed;
  section 5.2 when the activations are rotated too, each activation sub-block
              is transformed and then quantised at once (dynamic quantisation);
  section 5.4 eight 4-bit integers per 32-bit word; INT32 accumulation; the
              result is dequantised with the quantisation parameters.
  [Scholia] "Inference Quantization" notes, section 4: the symmetric INT4 grid
              is [-7, 7] with step absmax/7 (the worked example there).

Readings (each also in the design notes):
  * Y = X W^T with W stored [N][K]; the rotation acts on the contraction index
    K in groups of G consecutive columns: R = blockdiag(Hn, ..., Hn) with
    Hn = H_G / sqrt(G), H_G the Sylvester Hadamard matrix (H_1 = [1],
    H_2n = [[H_n, H_n], [H_n, -H_n]]). R R^T = I, so (X R)(W R)^T = X W^T;
    "multiply each sub-block by Hn" is the right product W[:, group] . Hn;
  * G is a power of two (16 ... 256; 128 by default) dividing K;
  * the rotated value of an fp16 row is r = fl32(fl32(S) * c_G) with
    S = x_group . H_G the EXACT +-1 sum (every partial sum of at most 256
    fp16 values is a multiple of 2^-24 below 2^24 in magnitude, so it is
    exact in float64 in any order) and c_G = fl32(1/sqrt(G)); for G a power of
    four c_G is a power of two and the second rounding is exact;
  * codes: q = clamp(rint(fl32(fl32(r * qmax) / a)), -qmax, qmax) with qmax =
    127 (W8A8) or 7 (W4A4), a the absmax of the quantisation group, rint half
    to even, a = 0 giving 0 (the same rule as the LLM.int8() path, with the
    product r * qmax rounded once because r is an fp32 value);
  * W8A8: no outlier split; per-token scales for the rotated X and per output
    row scales for the rotated W, over all K (the vector-wise scheme of the
    rest of the path; the page gives sub-block parameters for the W4A4 format);
  * W4A4: per sub-block scales: for the rotated X one absmax per (token, group
    of G columns), the 1 x G activation sub-block of dynamic quantisation; for
    the rotated W one absmax per G x G sub-block (G output rows by G columns);
    N is a multiple of G;
  * packing: code j of a run of eight along K sits in bits 4j..4j+3 of one
    uint32 (two's complement nibble, the lowest K index in the lowest nibble);
  * dequantisation: W8A8 Y = C * ax[m] * aw[n] / 127^2; W4A4
    Y = sum_g C_g * ax[m, g] * aw[n // G, g] / 7^2 with C_g the INT32 product
    over group g; both in float64, rounded once to fp16.

Parity status: every function is pinned by the CPU tests (Sylvester matrix
against the library routine, orthogonality, the preserved product and norm,
closed forms for a spike and a constant group, brute force on tiny inputs,
the INT4 example's grid, a hand-packed word, the per-row reduction of the
grouped dequantisation and the page's claim that rotation lowers the error
on inputs with outlier channels).
"""
from __future__ import annotations

import numpy as np

from .llm_int8 import absmax_codes, int32_gemm

QMAX_W8 = 127
QMAX_W4 = 7


def hadamard(G: int) -> np.ndarray:
    """The Sylvester Hadamard matrix H_G (entries +-1, int64), G a power of two."""
    if G < 1 or (G & (G - 1)) != 0:
        raise ValueError("G must be a power of two")
    H = np.ones((1, 1), dtype=np.int64)
    while H.shape[0] < G:
        H = np.block([[H, H], [H, -H]])
    return H


def rotation_scale(G: int) -> np.float32:
    """c_G = fl32(1/sqrt(G)), the normalisation of the regular Hadamard matrix."""
    return np.float32(1.0 / np.sqrt(float(G)))


def _check_groups(K: int, G: int):
    if G < 1 or (G & (G - 1)) != 0:
        raise ValueError("G must be a power of two")
    if K % G != 0:
        raise ValueError("K must be a multiple of G")


def hadamard_sums(X: np.ndarray, G: int) -> np.ndarray:
    """S[:, g*G + i] = sum_j X[:, g*G + j] * H_G[j, i], float64 [rows, K] (exact for fp16 X)."""
    Xf = np.asarray(X, dtype=np.float64)
    rows, K = Xf.shape
    _check_groups(K, G)
    H = hadamard(G).astype(np.float64)
    S = np.empty_like(Xf)
    for g in range(K // G):
        S[:, g * G:(g + 1) * G] = Xf[:, g * G:(g + 1) * G] @ H
    return S


def rotate_groups(X: np.ndarray, G: int) -> np.ndarray:
    """The rotated rows r = fl32(fl32(S) * c_G), float32 [rows, K]."""
    S = hadamard_sums(X, G)
    return S.astype(np.float32) * rotation_scale(G)


def rotate_groups_f64(X: np.ndarray, G: int) -> np.ndarray:
    """X . R in float64 (S / sqrt(G)), for the orthogonality checks."""
    return hadamard_sums(X, G) / np.sqrt(float(G))


# ---------------------------------------------------------------------------
# W8A8 after rotation: vector-wise scales (per token, per output row).
# ---------------------------------------------------------------------------
def quantize_rows_rotated(X: np.ndarray, G: int, qmax: int = QMAX_W8):
    """Rotate each row in groups of G, then one absmax per row over all K.

    Returns (codes int8 [rows, K], absmax fp32 [rows], r fp32 [rows, K])."""
    r = rotate_groups(X, G)
    a = np.max(np.abs(r), axis=1) if r.shape[1] else np.zeros(r.shape[0], np.float32)
    q = absmax_codes(r, a[:, None], qmax).astype(np.int8)
    return q, a.astype(np.float32), r


def rotated_w8a8_matmul(X: np.ndarray, Wq: np.ndarray, w_scale: np.ndarray, G: int):
    """The runtime W8A8 path with a weight already rotated and quantised by rows.

    Returns a dict with Y (fp16 [M, N]), Xq, x_scale, R (the rotated X) and C."""
    Xq, ax, r = quantize_rows_rotated(X, G, QMAX_W8)
    C = int32_gemm(Xq, Wq)
    Y64 = (np.asarray(C, np.float64) * np.asarray(ax, np.float64)[:, None]
           * np.asarray(w_scale, np.float64)[None, :] / float(QMAX_W8 * QMAX_W8))
    return dict(Y=Y64.astype(np.float16), Xq=Xq, x_scale=ax, R=r, C=C)


# ---------------------------------------------------------------------------
# W4A4 after rotation: per sub-block scales, eight codes per 32-bit word.
# ---------------------------------------------------------------------------
def quantize_act_groups(X: np.ndarray, G: int, qmax: int = QMAX_W4):
    """Rotate, then one absmax per (row, group of G columns).

    Returns (codes int8 [rows, K], absmax fp32 [rows, K/G], r fp32 [rows, K])."""
    r = rotate_groups(X, G)
    rows, K = r.shape
    a = np.abs(r).reshape(rows, K // G, G).max(axis=2) if K else np.zeros((rows, 0), np.float32)
    q = absmax_codes(r, np.repeat(a, G, axis=1), qmax).astype(np.int8)
    return q, a.astype(np.float32), r


def quantize_weight_blocks(W: np.ndarray, G: int, qmax: int = QMAX_W4):
    """Rotate the rows of W [N, K], then one absmax per G x G sub-block.

    Returns (codes int8 [N, K], absmax fp32 [N/G, K/G], r fp32 [N, K])."""
    N = np.asarray(W).shape[0]
    if N % G != 0:
        raise ValueError("N must be a multiple of G")
    r = rotate_groups(W, G)
    K = r.shape[1]
    a = np.abs(r).reshape(N // G, G, K // G, G).max(axis=(1, 3))
    full = np.repeat(np.repeat(a, G, axis=0), G, axis=1)
    q = absmax_codes(r, full, qmax).astype(np.int8)
    return q, a.astype(np.float32), r


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Codes in [-8, 7], int [rows, K] (K % 8 == 0) -> uint32 [rows, K/8]."""
    q = np.asarray(q, dtype=np.int64)
    rows, K = q.shape
    if K % 8 != 0:
        raise ValueError("K must be a multiple of 8")
    if np.any(q < -8) or np.any(q > 7):
        raise ValueError("code outside the 4-bit range")
    nib = (q & 0xF).reshape(rows, K // 8, 8).astype(np.uint64)
    shifts = (4 * np.arange(8, dtype=np.uint64))[None, None, :]
    return np.bitwise_or.reduce(nib << shifts, axis=2).astype(np.uint32)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    """uint32 [rows, K/8] -> int8 codes [rows, K] (sign-extended nibbles)."""
    p = np.asarray(p, dtype=np.uint64)
    rows, W = p.shape
    shifts = (4 * np.arange(8, dtype=np.uint64))[None, None, :]
    nib = ((p[:, :, None] >> shifts) & 0xF).astype(np.int64)
    return np.where(nib >= 8, nib - 16, nib).reshape(rows, 8 * W).astype(np.int8)


def group_gemm(Xq: np.ndarray, Wq: np.ndarray, G: int) -> np.ndarray:
    """C_g[g, m, n] = sum_{k in group g} Xq[m, k] Wq[n, k], exact, int32 [K/G, M, N]."""
    K = np.asarray(Xq).shape[1]
    _check_groups(K, G)
    return np.stack([int32_gemm(Xq[:, g * G:(g + 1) * G], Wq[:, g * G:(g + 1) * G])
                     for g in range(K // G)]) if K else np.zeros((0, Xq.shape[0], Wq.shape[0]), np.int32)


def dequantize_groups(Cg: np.ndarray, ax: np.ndarray, aw: np.ndarray, G: int,
                      qmax: int = QMAX_W4) -> np.ndarray:
    """float64 Y[m, n] = sum_g Cg[g, m, n] * ax[m, g] * aw[n // G, g] / qmax^2."""
    Cg = np.asarray(Cg, np.float64)
    ax = np.asarray(ax, np.float64)
    awn = np.repeat(np.asarray(aw, np.float64), G, axis=0)      # [N, K/G]
    Y = np.zeros(Cg.shape[1:], np.float64)
    for g in range(Cg.shape[0]):
        Y += Cg[g] * ax[:, g][:, None] * awn[:, g][None, :]
    return Y / float(qmax * qmax)


def rotated_w4a4_matmul(X: np.ndarray, Wp: np.ndarray, aw: np.ndarray, G: int):
    """The runtime W4A4 path with a weight already rotated, block-quantised and packed.

    Returns a dict with Y (fp16 [M, N]), Xp (packed codes uint32 [M, K/8]),
    Xq (int8 codes), x_scale (fp32 [M, K/G]) and Cg (int32 [K/G, M, N])."""
    Xq, ax, _ = quantize_act_groups(X, G, QMAX_W4)
    Wq = unpack_int4(Wp)
    Cg = group_gemm(Xq, Wq, G)
    Y64 = dequantize_groups(Cg, ax, aw, G, QMAX_W4)
    return dict(Y=Y64.astype(np.float16), Xp=pack_int4(Xq), Xq=Xq, x_scale=ax, Cg=Cg)
