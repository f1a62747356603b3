"""CPU oracle for the LLM.int8() mixed-precision decomposition matmul Y = X.W^T.

TEST INFRASTRUCTURE ONLY. The oracle itself is the plain C++17 program
llm_int8.cpp next to this file (compiled by oracle/build.py into
liborc_llm_int8.so, with -ffp-contract=off and no -ffast-math). This module
is its ctypes shim: each function below checks and converts its numpy
arguments, allocates the outputs and calls the C++ function of the same name;
every step of the method's arithmetic runs in the C++ code. Only the tests,
the smoke check and the benchmark's CPU legs may import this module; the
product path never does, and neither side shares code with the other.

Sources and readings are stated in llm_int8.cpp's header:
  [AIInfra]    Infrasys-AI/AIInfra "05Infer/06CompDistill/05Quantization01",
               LLM.int8() section (detection, vector-wise absmax INT8, INT32
               accumulation, outer-product dequantisation, FP16 outlier
               product, final sum; training notes on the top 1-2% dimensions);
  [Scholia]    scholia-log "Inference Quantization", sections 4 and 6;
  [Tanjunchen] "quantization explained part 2", sections 1.2 and 4.5.

The environment variable LLM_INT8_ORACLE_LIB points the shim at another build
of the oracle (the planted-mistake tests use it); ORACLE_THREADS sets the
number of C++ threads (default: one per hardware thread).

Parity status: every function is pinned by the CPU tests.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

QMAX_INT8 = 127
ZP_QMIN, ZP_QMAX = -128, 127

_c_p = ctypes.c_void_p
_c_i = ctypes.c_int
_c_i64 = ctypes.c_int64
_c_f = ctypes.c_float

_PROTOS = {
    "orc_threads": (_c_i, []),
    "orc_set_threads": (None, [_c_i]),
    "orc_half_to_float": (None, [_c_p, _c_i64, _c_p]),
    "orc_double_to_half": (None, [_c_p, _c_i64, _c_p]),
    "orc_absmax_codes": (None, [_c_p, _c_p, _c_i64, _c_i, _c_p]),
    "orc_absmax": (_c_f, [_c_p, _c_i64]),
    "orc_dequantize_codes": (None, [_c_p, _c_p, _c_i64, _c_i, _c_p]),
    "orc_quantize_weight_rows": (None, [_c_p, _c_i, _c_i, _c_p, _c_p]),
    "orc_find_outlier_cols": (_c_i, [_c_p, _c_i, _c_i, _c_f, _c_p]),
    "orc_mask_to_bitmap": (_c_i, [_c_p, _c_i, _c_p, _c_p]),
    "orc_find_topk_cols": (None, [_c_p, _c_i, _c_i, _c_i, _c_p]),
    "orc_quantize_act_rows": (None, [_c_p, _c_i, _c_i, _c_p, _c_p, _c_p]),
    "orc_quantize_act_rows_zp": (None, [_c_p, _c_i, _c_i, _c_p, _c_p, _c_p, _c_p]),
    "orc_int32_gemm": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_p]),
    "orc_weight_rowsum": (None, [_c_p, _c_i, _c_i, _c_p]),
    "orc_dequantize": (None, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_p]),
    "orc_dequantize_zp": (None, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_p]),
    "orc_outlier_gemm": (None, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_p, _c_i, _c_p]),
    "orc_sum_to_half": (None, [_c_p, _c_p, _c_i64, _c_p]),
    "orc_llm_int8_matmul": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_f, _c_p, _c_p, _c_p, _c_i,
                                   _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                                   _c_p]),
    "orc_llm_int8_matmul_at": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_f, _c_p,
                                      _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p]),
}

_LIB = None


def lib():
    """The loaded C++ oracle (built first if missing or older than its source)."""
    global _LIB
    if _LIB is None:
        path = os.environ.get("LLM_INT8_ORACLE_LIB")
        if not path:
            from . import build as _build
            path = _build.build()
        L = ctypes.CDLL(path)
        for name, (res, args) in _PROTOS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def threads() -> int:
    """Threads the C++ oracle runs on."""
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


# --------------------------------------------------------------------------- marshalling
def _ptr(a):
    return a.ctypes.data_as(_c_p) if a is not None else None


def _out(shape, dtype):
    return np.empty(shape, dtype=dtype)


def _half_bits(a, name="X"):
    """A C-contiguous uint16 view of the binary16 values of `a` (2-D).

    Float16 arrays pass as they are; other float arrays are accepted only if
    every value is exactly a binary16 value (the inputs of this path are fp16).
    """
    a = np.asarray(a)
    if a.dtype != np.float16:
        h = a.astype(np.float16)
        if not np.array_equal(h.astype(a.dtype), a):
            raise ValueError(f"{name} must hold binary16 values")
        a = h
    return np.ascontiguousarray(a).view(np.uint16)


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _mask(mask, K):
    m = np.ascontiguousarray(np.asarray(mask, dtype=bool)).view(np.uint8)
    if m.size != K:
        raise ValueError("mask size must equal K")
    return m


# --------------------------------------------------------------------------- binary16
def half_to_float(h):
    """binary16 values (fp16 array) -> float32, decoded by the C++ oracle."""
    b = _half_bits(np.asarray(h, np.float16).reshape(-1), "h")
    out = _out(b.size, np.float32)
    lib().orc_half_to_float(_ptr(b), b.size, _ptr(out))
    return out.reshape(np.shape(h))


def double_to_half(d):
    """float64 -> nearest binary16 (ties to even), rounded once by the C++ oracle."""
    d64 = np.ascontiguousarray(np.asarray(d, dtype=np.float64))
    out = _out(d64.shape, np.uint16)
    lib().orc_double_to_half(_ptr(d64), d64.size, _ptr(out))
    return out.view(np.float16).reshape(np.shape(d))


# --------------------------------------------------------------------------- quantiser
def absmax_codes(x, absmax, qmax: int) -> np.ndarray:
    """Integer codes clamp(rint((x*qmax)/absmax), -qmax, qmax) as int32.

    `x` is taken as float32 and `absmax` broadcasts against it; an absmax of 0
    gives code 0 ([Scholia] section 4: an all-zero group is handled apart).
    """
    x32 = _f32(x)
    a32 = np.ascontiguousarray(np.broadcast_to(np.asarray(absmax, dtype=np.float32), x32.shape))
    q = _out(x32.shape, np.int32)
    lib().orc_absmax_codes(_ptr(x32), _ptr(a32), x32.size, int(qmax), _ptr(q))
    return q.reshape(np.shape(x))


def quantize_per_tensor(x, qmax: int):
    """One scale for the whole tensor: (codes, absmax). [Scholia] section 4."""
    x32 = _f32(x)
    a = np.float32(lib().orc_absmax(_ptr(x32), x32.size))
    return absmax_codes(x32, a, qmax), a


def step_size(absmax, qmax: int) -> np.ndarray:
    """Width of one integer step in real units, s = absmax/qmax ([Scholia] s4), float64."""
    a = np.ascontiguousarray(np.asarray(absmax, dtype=np.float64))
    out = _out(a.shape, np.float64)
    lib().orc_dequantize_codes(None, _ptr(a), a.size, int(qmax), _ptr(out))
    return out.reshape(np.shape(absmax))


def dequantize_codes(q, absmax, qmax: int) -> np.ndarray:
    """x_hat = s*q with s = absmax/qmax ([Scholia] section 4), in float64."""
    q32 = np.asarray(q, dtype=np.int32)
    shape = np.broadcast_shapes(q32.shape, np.shape(absmax))
    qb = np.ascontiguousarray(np.broadcast_to(q32, shape))
    ab = np.ascontiguousarray(np.broadcast_to(np.asarray(absmax, dtype=np.float64), shape))
    out = _out(qb.shape, np.float64)
    lib().orc_dequantize_codes(_ptr(qb), _ptr(ab), qb.size, int(qmax), _ptr(out))
    return out.reshape(shape)


# --------------------------------------------------------------------------- the path's steps
def quantize_weight_rows(W):
    """W fp16 [N, K] -> (Wq int8 [N, K], w_scale fp32 [N] = row absmax over all K)."""
    Wb = _half_bits(W, "W")
    N, K = Wb.shape
    Wq = _out((N, K), np.int8)
    aw = _out(N, np.float32)
    lib().orc_quantize_weight_rows(_ptr(Wb), N, K, _ptr(Wq), _ptr(aw))
    return Wq, aw


def mask_to_bitmap(mask):
    """(bitmap uint32[ceil(K/32)], count, idx int32 ascending) of a boolean column mask."""
    m = np.ascontiguousarray(np.asarray(mask, dtype=bool)).view(np.uint8).reshape(-1)
    K = m.size
    bitmap = _out((K + 31) // 32, np.uint32)
    idx = _out(max(K, 1), np.int32)
    count = lib().orc_mask_to_bitmap(_ptr(m), K, _ptr(bitmap), _ptr(idx))
    return bitmap, int(count), idx[:count].copy()


def find_outlier_cols(X, threshold: float):
    """Returns (mask bool[K], bitmap uint32[ceil(K/32)], count, idx int32 ascending).

    Column j is an outlier iff |X[i, j]| > threshold (binary32) for some row i.
    """
    Xb = _half_bits(X)
    M, K = Xb.shape
    mask = _out(K, np.uint8)
    lib().orc_find_outlier_cols(_ptr(Xb), M, K, float(threshold), _ptr(mask))
    mask = mask.astype(bool)
    bitmap, count, idx = mask_to_bitmap(mask)
    return mask, bitmap, count, idx


def find_topk_cols(X, k: int) -> np.ndarray:
    """Mask (bool [K]) of the k columns with the largest max |x| over the rows
    (ties to the lower index, k clipped to [0, K]); [AIInfra] training notes."""
    Xb = _half_bits(X)
    M, K = Xb.shape
    mask = _out(K, np.uint8)
    lib().orc_find_topk_cols(_ptr(Xb), M, K, int(max(0, min(int(k), K))), _ptr(mask))
    return mask.astype(bool)


def quantize_act_rows(X, outlier_mask):
    """X fp16 [M, K] -> (Xq int8 [M, K] with 0 at outlier columns, x_scale fp32 [M])."""
    Xb = _half_bits(X)
    M, K = Xb.shape
    m = _mask(outlier_mask, K)
    Xq = _out((M, K), np.int8)
    ax = _out(M, np.float32)
    lib().orc_quantize_act_rows(_ptr(Xb), M, K, _ptr(m), _ptr(Xq), _ptr(ax))
    return Xq, ax


def quantize_act_rows_zp(X, outlier_mask):
    """Per-token zero-point INT8 codes of the non-outlier columns ([Scholia] s6).

    Returns (Xq int8 [M, K], step fp32 [M], zero int32 [M]); see llm_int8.cpp.
    """
    Xb = _half_bits(X)
    M, K = Xb.shape
    m = _mask(outlier_mask, K)
    Xq = _out((M, K), np.int8)
    step = _out(M, np.float32)
    zero = _out(M, np.int32)
    lib().orc_quantize_act_rows_zp(_ptr(Xb), M, K, _ptr(m), _ptr(Xq), _ptr(step), _ptr(zero))
    return Xq, step, zero


def int32_gemm(Xq, Wq) -> np.ndarray:
    """C[i, n] = sum_k Xq[i, k] * Wq[n, k], exact, as int32 (asserted to fit)."""
    A = np.ascontiguousarray(np.asarray(Xq, dtype=np.int8))
    B = np.ascontiguousarray(np.asarray(Wq, dtype=np.int8))
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K
    C = _out((M, N), np.int32)
    assert lib().orc_int32_gemm(_ptr(A), _ptr(B), M, N, K, _ptr(C)) == 0, "int32 overflow"
    return C


def weight_rowsum(Wq) -> np.ndarray:
    """sum_k Wq[n, k] (int32 [N]), the zero-point correction's weight factor."""
    B = np.ascontiguousarray(np.asarray(Wq, dtype=np.int8))
    N, K = B.shape
    s = _out(N, np.int32)
    lib().orc_weight_rowsum(_ptr(B), N, K, _ptr(s))
    return s


def dequantize(C, x_scale, w_scale) -> np.ndarray:
    """float64 C_normal[i, n] = C[i, n] * x_scale[i] * w_scale[n] / 127^2."""
    C32 = np.ascontiguousarray(np.asarray(C, dtype=np.int32))
    M, N = C32.shape
    xs, ws = _f32(x_scale), _f32(w_scale)
    out = _out((M, N), np.float64)
    lib().orc_dequantize(_ptr(C32), _ptr(xs), _ptr(ws), M, N, _ptr(out))
    return out


def dequantize_zp(C, zero, step, wsum, w_scale) -> np.ndarray:
    """step*w_scale/127*(C - zero*wsum), float64."""
    C32 = np.ascontiguousarray(np.asarray(C, dtype=np.int32))
    M, N = C32.shape
    z = np.ascontiguousarray(np.asarray(zero, dtype=np.int32))
    s = np.ascontiguousarray(np.asarray(wsum, dtype=np.int32))
    out = _out((M, N), np.float64)
    lib().orc_dequantize_zp(_ptr(C32), _ptr(z), _ptr(_f32(step)), _ptr(s), _ptr(_f32(w_scale)),
                            M, N, _ptr(out))
    return out


def outlier_gemm(X, W, idx) -> np.ndarray:
    """float64 C_outlier[i, n] = sum_{j in O} X[i, j] * W[n, j] over the list idx."""
    Xb, Wb = _half_bits(X), _half_bits(W, "W")
    M, K = Xb.shape
    N = Wb.shape[0]
    ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
    out = _out((M, N), np.float64)
    lib().orc_outlier_gemm(_ptr(Xb), _ptr(Wb), M, N, K, _ptr(ix), ix.size, _ptr(out))
    return out


# --------------------------------------------------------------------------- whole path
def llm_int8_matmul(X, W, threshold: float = 6.0, Wq=None, w_scale=None, outlier_mask=None,
                    zeropoint: bool = False, intermediates: bool = True):
    """All steps of the path; returns a dict with Y (fp16 [M, N]) and the intermediates.

    `W` is the fp16 weight [N, K]; it supplies the outlier columns of the FP16
    product. `Wq`/`w_scale` default to quantize_weight_rows(W). `outlier_mask`
    (bool [K]) replaces the detection step with a given outlier set (the set
    of a batch whose tokens are split over several processes; [AIInfra]: O is
    a property of the batch's activations); the threshold is then unused.
    `zeropoint` quantises the non-outlier part of each token with a zero point
    instead of the symmetric absmax; x_scale then holds the step and the
    result also has `zero` and `wsum`. With `intermediates=False` the M x N
    intermediates (C, C_normal, C_outlier) are not returned.
    """
    Xb, Wb = _half_bits(X), _half_bits(W, "W")
    M, K = Xb.shape
    N = Wb.shape[0]
    assert Wb.shape[1] == K
    if Wq is None or w_scale is None:
        Wq, w_scale = quantize_weight_rows(W)
    Wq = np.ascontiguousarray(np.asarray(Wq, dtype=np.int8))
    w_scale = _f32(w_scale)
    mask_in = None if outlier_mask is None else _mask(outlier_mask, K)
    mask = _out(K, np.uint8)
    bitmap = _out((K + 31) // 32, np.uint32)
    idx = _out(max(K, 1), np.int32)
    Xq = _out((M, K), np.int8)
    x_scale = _out(M, np.float32)
    zero = _out(M, np.int32) if zeropoint else None
    wsum = _out(N, np.int32) if zeropoint else None
    C = _out((M, N), np.int32) if intermediates else None
    Cn = _out((M, N), np.float64) if intermediates else None
    Co = _out((M, N), np.float64) if intermediates else None
    Y = _out((M, N), np.uint16)
    count = lib().orc_llm_int8_matmul(
        _ptr(Xb), _ptr(Wb), M, N, K, float(threshold), _ptr(Wq), _ptr(w_scale), _ptr(mask_in),
        1 if zeropoint else 0, _ptr(mask), _ptr(bitmap), _ptr(idx), _ptr(Xq), _ptr(x_scale),
        _ptr(zero), _ptr(wsum), _ptr(C), _ptr(Cn), _ptr(Co), _ptr(Y))
    assert count >= 0, "int32 overflow"
    res = dict(Y=Y.view(np.float16), mask=mask.astype(bool), bitmap=bitmap, count=int(count),
               idx=idx[:count].copy(), Xq=Xq, x_scale=x_scale, Wq=Wq, w_scale=w_scale)
    if intermediates:
        res.update(C=C, C_normal=Cn, C_outlier=Co)
    if zeropoint:
        res.update(zero=zero, wsum=wsum)
    return res


def llm_int8_matmul_at(X, W, Wq, w_scale, threshold: float, rows, cols):
    """Y[rows[t], cols[t]] for sampled output positions, one by one.

    Detection runs over the whole X (the outlier set depends on every row);
    only the sampled rows are quantised and only the sampled outputs formed.
    Returns (Y_samples fp16, C_samples int32, mask, x_scale of the sampled rows).
    """
    Xb, Wb = _half_bits(X), _half_bits(W, "W")
    M, K = Xb.shape
    N = Wb.shape[0]
    Wq = np.ascontiguousarray(np.asarray(Wq, dtype=np.int8))
    ws = _f32(w_scale)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    c = np.ascontiguousarray(np.asarray(cols, dtype=np.int64).reshape(-1))
    assert r.size == c.size
    assert r.size == 0 or (r.min() >= 0 and r.max() < M and c.min() >= 0 and c.max() < N)
    mask = _out(K, np.uint8)
    Y = _out(r.size, np.uint16)
    C = _out(r.size, np.int32)
    xs = _out(r.size, np.float32)
    lib().orc_llm_int8_matmul_at(_ptr(Xb), _ptr(Wb), _ptr(Wq), _ptr(ws), M, N, K,
                                 float(threshold), _ptr(r), _ptr(c), r.size, _ptr(mask), _ptr(Y),
                                 _ptr(C), _ptr(xs))
    return Y.view(np.float16), C, mask.astype(bool), xs
