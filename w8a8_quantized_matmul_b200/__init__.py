"""LLM.int8() mixed-precision decomposition matmul for B200 (sm_100a).

Thin Python binding over the C ABI of libint8mm (include/int8mm.h). Each
function has the name of the C entry point it calls; PyTorch supplies only
device memory and the current CUDA stream, and every step of the path runs
in the library's CUDA kernels. There is no CPU fallback: calling any compute
entry point without the built library or without a B200 raises.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import (  # noqa: F401
    I8MM_ERR_ALIGNMENT,
    I8MM_ERR_CUDA,
    I8MM_ERR_INVALID_ARG,
    I8MM_ERR_TIMEOUT,
    I8MM_ERR_UNSUPPORTED_DEVICE,
    I8MM_ERR_WORKSPACE,
    I8MM_OK,
    Int8mmError,
    WorkspaceLayout,
    check,
    load,
    status_string,
)

__all__ = [
    "int8_quantize_weight_rows",
    "int8_transpose_weight",
    "int8_find_outlier_cols",
    "int8_quantize_act_rows",
    "int8_mixed_matmul_workspace_size",
    "int8_mixed_matmul_workspace_layout",
    "int8_mixed_matmul",
    "int8_mixed_matmul_profiled",
    "int8_mixed_matmul_stage",
    "int8_mixed_matmul_sharded",
    "int8_debug_gemm_i32",
    "int8_column_absmax",
    "int8_mixed_matmul_topk",
    "int8_weight_rowsum",
    "int8_mixed_matmul_zp",
    "int8_smoothquant_factors",
    "int8_smoothquant_weight_rows",
    "int8_smoothquant_workspace_size",
    "int8_smoothquant_matmul",
    "int8_device_status",
    "Int8mmError",
]


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def int8_quantize_weight_rows(W, Wq=None, w_scale=None, stream=None):
    """W fp16 [N, K] -> (Wq int8 [N, K], w_scale fp32 [N] row absmax)."""
    N, K = W.shape
    _need(W, "W", torch.float16, (N, K))
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    w_scale = torch.empty((N,), dtype=torch.float32, device=W.device) if w_scale is None else w_scale
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    check("int8_quantize_weight_rows",
          load().int8_quantize_weight_rows(_ptr(W), N, K, _ptr(Wq), _ptr(w_scale), _stream(stream)))
    return Wq, w_scale


def int8_transpose_weight(W, Wt=None, stream=None):
    """W fp16 [N, K] -> Wt fp16 [K, N] (offline layout of the fp16 weight that the
    mixed-matmul calls read the outlier features from)."""
    N, K = W.shape
    _need(W, "W", torch.float16, (N, K))
    Wt = torch.empty((K, N), dtype=torch.float16, device=W.device) if Wt is None else Wt
    _need(Wt, "Wt", torch.float16, (K, N))
    check("int8_transpose_weight", load().int8_transpose_weight(_ptr(W), N, K, _ptr(Wt), _stream(stream)))
    return Wt


def int8_find_outlier_cols(X, threshold=6.0, col_bitmap=None, n_outliers=None, col_idx=None,
                           stream=None):
    """X fp16 [M, K] -> (bitmap uint32-as-int32 [ceil(K/32)], count int32 [1], col_idx int32 [K])."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    words = (K + 31) // 32
    dev = X.device
    col_bitmap = torch.empty((words,), dtype=torch.int32, device=dev) if col_bitmap is None else col_bitmap
    n_outliers = torch.empty((4,), dtype=torch.int32, device=dev)[:1] if n_outliers is None else n_outliers
    col_idx = torch.empty((K,), dtype=torch.int32, device=dev) if col_idx is None else col_idx
    _need(col_bitmap, "col_bitmap", torch.int32, (words,))
    _need(col_idx, "col_idx", torch.int32, (K,))
    check("int8_find_outlier_cols",
          load().int8_find_outlier_cols(_ptr(X), M, K, float(threshold), _ptr(col_bitmap),
                                        _ptr(n_outliers), _ptr(col_idx), _stream(stream)))
    return col_bitmap, n_outliers, col_idx


def int8_quantize_act_rows(X, col_bitmap, Xq=None, x_scale=None, stream=None):
    """X fp16 [M, K] + outlier bitmap -> (Xq int8 [M, K], x_scale fp32 [M])."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    _need(col_bitmap, "col_bitmap", torch.int32, ((K + 31) // 32,))
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    x_scale = torch.empty((M,), dtype=torch.float32, device=X.device) if x_scale is None else x_scale
    _need(Xq, "Xq", torch.int8, (M, K))
    _need(x_scale, "x_scale", torch.float32, (M,))
    check("int8_quantize_act_rows",
          load().int8_quantize_act_rows(_ptr(X), M, K, _ptr(col_bitmap), _ptr(Xq), _ptr(x_scale),
                                        _stream(stream)))
    return Xq, x_scale


def int8_mixed_matmul_workspace_size(M: int, N: int, K: int) -> int:
    return int(load().int8_mixed_matmul_workspace_size(M, N, K))


def int8_mixed_matmul_workspace_layout(M: int, N: int, K: int) -> WorkspaceLayout:
    lay = WorkspaceLayout()
    check("int8_mixed_matmul_workspace_layout",
          load().int8_mixed_matmul_workspace_layout(M, N, K, ctypes.byref(lay)))
    return lay


def int8_mixed_matmul(X, Wq, w_scale, Wt_fp16, threshold=6.0, Y=None, workspace=None, stream=None):
    """Y = LLM.int8() decomposition of X . W^T; returns (Y fp16 [M, N], workspace uint8)."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    _need(Wt_fp16, "Wt_fp16", torch.float16, (K, N))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int8_mixed_matmul_workspace_size(M, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_mixed_matmul",
          load().int8_mixed_matmul(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(Wt_fp16), M, N, K,
                                   float(threshold), _ptr(Y), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y, workspace


def int8_mixed_matmul_profiled(X, Wq, w_scale, Wt_fp16, threshold, Y, workspace, events,
                               stream=None):
    """int8_mixed_matmul that also records three torch.cuda.Event objects on the stream:
    before the call, between the quantisation stage and the GEMM, and after the GEMM."""
    M, K = X.shape
    N = Wq.shape[0]
    s = torch.cuda.current_stream() if stream is None else stream
    handles = []
    for ev in events:
        if not ev.cuda_event:
            ev.record(s)   # torch creates the underlying cudaEvent_t lazily
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * 3)(*handles)
    check("int8_mixed_matmul_profiled",
          load().int8_mixed_matmul_profiled(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(Wt_fp16), M, N, K,
                                            float(threshold), _ptr(Y), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            ctypes.c_void_p(s.cuda_stream), arr))
    return Y


def int8_mixed_matmul_stage(stage, X, Wq, w_scale, Wt_fp16, threshold, Y, workspace, stream=None):
    """One stage of int8_mixed_matmul (1: quantisation kernel, 2: GEMM kernel) for timing."""
    M, K = X.shape
    N = Wq.shape[0]
    check("int8_mixed_matmul_stage",
          load().int8_mixed_matmul_stage(int(stage), _ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(Wt_fp16),
                                         M, N, K, float(threshold), _ptr(Y), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))
    return Y


def int8_mixed_matmul_sharded(X, Wq, w_scale, Wt_fp16, bitmaps, Y=None, workspace=None,
                              stream=None):
    """One rank's part of a token-sharded int8_mixed_matmul.

    X fp16 [M, K] are this rank's tokens; bitmaps int32 [n, ceil(K/32)] are the
    outlier bitmaps of all ranks' int8_find_outlier_cols (the outlier set is their
    OR). Returns (Y fp16 [M, N], workspace)."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    _need(Wt_fp16, "Wt_fp16", torch.float16, (K, N))
    words = (K + 31) // 32
    if bitmaps.dim() != 2:
        raise ValueError("bitmaps must be [n_ranks, ceil(K/32)]")
    _need(bitmaps, "bitmaps", torch.int32, (bitmaps.shape[0], words))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int8_mixed_matmul_workspace_size(M, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_mixed_matmul_sharded",
          load().int8_mixed_matmul_sharded(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(Wt_fp16), M, N,
                                           K, _ptr(bitmaps), int(bitmaps.shape[0]), _ptr(Y),
                                           _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)))
    return Y, workspace


def int8_mixed_matmul_topk(X, Wq, w_scale, Wt_fp16, k, Y=None, workspace=None, stream=None):
    """LLM.int8() matmul whose outlier set is the k columns of largest max |x|.
    Returns (Y fp16 [M, N], workspace); workspace_views() reads the intermediates."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    _need(Wt_fp16, "Wt_fp16", torch.float16, (K, N))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int(load().int8_mixed_matmul_topk_workspace_size(M, N, K))
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_mixed_matmul_topk",
          load().int8_mixed_matmul_topk(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(Wt_fp16), M, N, K,
                                        int(k), _ptr(Y), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))
    return Y, workspace


def int8_weight_rowsum(Wq, rowsum=None, stream=None):
    """sum_k Wq[n, k] as int32 [N] (the zero-point correction's weight factor)."""
    N, K = Wq.shape
    _need(Wq, "Wq", torch.int8, (N, K))
    rowsum = torch.empty((N,), dtype=torch.int32, device=Wq.device) if rowsum is None else rowsum
    check("int8_weight_rowsum",
          load().int8_weight_rowsum(_ptr(Wq), N, K, _ptr(rowsum), _stream(stream)))
    return rowsum


def int8_mixed_matmul_zp(X, Wq, w_scale, w_rowsum, Wt_fp16, threshold=6.0, Y=None,
                         workspace=None, stream=None):
    """The decomposition with zero-point codes for the non-outlier part.
    Returns (Y fp16 [M, N], workspace); zero points via zeropoint_views()."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    _need(w_rowsum, "w_rowsum", torch.int32, (N,))
    _need(Wt_fp16, "Wt_fp16", torch.float16, (K, N))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int(load().int8_mixed_matmul_zp_workspace_size(M, N, K))
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_mixed_matmul_zp",
          load().int8_mixed_matmul_zp(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(w_rowsum),
                                      _ptr(Wt_fp16), M, N, K, float(threshold), _ptr(Y),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)))
    return Y, workspace


def zeropoint_views(workspace: torch.Tensor, M: int, N: int, K: int) -> torch.Tensor:
    """The int32 [M] zero points int8_mixed_matmul_zp leaves after the regular layout."""
    off = (int8_mixed_matmul_workspace_size(M, N, K) + 255) // 256 * 256
    return workspace[off:off + 4 * M].view(torch.int32)


def int8_column_absmax(X, colmax=None, stream=None):
    """Running column max |x| of fp16 [rows, K] into fp32 colmax [K] (zeros if None)."""
    rows, K = X.shape
    _need(X, "X", torch.float16, (rows, K))
    colmax = torch.zeros((K,), dtype=torch.float32, device=X.device) if colmax is None else colmax
    _need(colmax, "colmax", torch.float32, (K,))
    check("int8_column_absmax",
          load().int8_column_absmax(_ptr(X), rows, K, _ptr(colmax), _stream(stream)))
    return colmax


def int8_smoothquant_factors(act_absmax, w_absmax, alpha=0.5, s=None, s_rcp=None, stream=None):
    """SmoothQuant factors s [K] and their reciprocals fl32(1/s) [K]."""
    K = act_absmax.numel()
    _need(act_absmax, "act_absmax", torch.float32, (K,))
    _need(w_absmax, "w_absmax", torch.float32, (K,))
    s = torch.empty((K,), dtype=torch.float32, device=act_absmax.device) if s is None else s
    s_rcp = torch.empty_like(s) if s_rcp is None else s_rcp
    check("int8_smoothquant_factors",
          load().int8_smoothquant_factors(_ptr(act_absmax), _ptr(w_absmax), K, float(alpha),
                                          _ptr(s), _ptr(s_rcp), _stream(stream)))
    return s, s_rcp


def int8_smoothquant_weight_rows(W, s, Wq=None, w_scale=None, stream=None):
    """fp16 W [N, K] and factors s [K] -> (Wq int8 [N, K], w_scale fp32 [N]) of W * s."""
    N, K = W.shape
    _need(W, "W", torch.float16, (N, K))
    _need(s, "s", torch.float32, (K,))
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    w_scale = torch.empty((N,), dtype=torch.float32, device=W.device) if w_scale is None else w_scale
    check("int8_smoothquant_weight_rows",
          load().int8_smoothquant_weight_rows(_ptr(W), _ptr(s), N, K, _ptr(Wq), _ptr(w_scale),
                                              _stream(stream)))
    return Wq, w_scale


def int8_smoothquant_workspace_size(M: int, N: int, K: int) -> int:
    return int(load().int8_smoothquant_workspace_size(M, N, K))


def int8_smoothquant_matmul(X, Wq, w_scale, s_rcp, Y=None, workspace=None, stream=None):
    """SmoothQuant W8A8 runtime path; returns (Y fp16 [M, N], workspace)."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    _need(s_rcp, "s_rcp", torch.float32, (K,))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int8_smoothquant_workspace_size(M, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_smoothquant_matmul",
          load().int8_smoothquant_matmul(_ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(s_rcp), M, N, K,
                                         _ptr(Y), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))
    return Y, workspace


def smoothquant_workspace_views(workspace: torch.Tensor, M: int, K: int) -> dict:
    """x_scale fp32 [M] and Xq int8 [M, K] that int8_smoothquant_matmul leaves in its workspace."""
    def up(x):
        return (x + 255) // 256 * 256
    xs_off = up(16)
    xq_off = up(xs_off + 4 * M)
    return dict(status=workspace[0:4].view(torch.int32),
                x_scale=workspace[xs_off:xs_off + 4 * M].view(torch.float32),
                Xq=workspace[xq_off:xq_off + M * K].view(torch.int8).view(M, K))


def int8_debug_gemm_i32(Xq, Wq, C=None, stream=None):
    """C int32 [M, N] = Xq . Wq^T on the tensor-core kernel (test hook)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    _need(Xq, "Xq", torch.int8, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    C = torch.empty((M, N), dtype=torch.int32, device=Xq.device) if C is None else C
    _need(C, "C", torch.int32, (M, N))
    check("int8_debug_gemm_i32",
          load().int8_debug_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(C), _stream(stream)))
    return C


def int8_device_status(workspace, stream=None) -> int:
    """Device status word left by the last int8_mixed_matmul in `workspace` (syncs)."""
    return int(load().int8_device_status(_ptr(workspace), _stream(stream)))


def workspace_views(workspace: torch.Tensor, M: int, N: int, K: int) -> dict:
    """Tensor views of the intermediates int8_mixed_matmul leaves in its workspace."""
    lay = int8_mixed_matmul_workspace_layout(M, N, K)
    words = (K + 31) // 32
    ld = lay.panel_ld

    def view(off, nbytes, dtype, shape):
        return workspace[off:off + nbytes].view(dtype).view(shape)

    return dict(
        n_outliers=view(lay.n_outliers, 4, torch.int32, (1,)),
        status=view(lay.status, 4, torch.int32, (1,)),
        col_bitmap=view(lay.col_bitmap, 4 * words, torch.int32, (words,)),
        col_idx=view(lay.col_idx, 4 * K, torch.int32, (K,)),
        x_scale=view(lay.x_scale, 4 * M, torch.float32, (M,)),
        Xq=view(lay.Xq, M * K, torch.int8, (M, K)),
        X_O=view(lay.X_O, 2 * M * ld, torch.float16, (M, ld)),
        W_O=view(lay.W_O, 2 * N * ld, torch.float16, (N, ld)),
    )


# --------------------------------------------------------------- grouped Hadamard rotation
def int8_rotate_quantize_rows(X, G=128, Xq=None, absmax=None, R=None, stream=None):
    """Rotate each row of X fp16 [rows, K] in groups of G, per-row absmax INT8 codes.
    Returns (Xq int8 [rows, K], absmax fp32 [rows]); R (fp32 [rows, K]) if given
    receives the rotated values."""
    rows, K = X.shape
    _need(X, "X", torch.float16, (rows, K))
    Xq = torch.empty((rows, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    absmax = torch.empty((rows,), dtype=torch.float32, device=X.device) if absmax is None else absmax
    _need(Xq, "Xq", torch.int8, (rows, K))
    _need(absmax, "absmax", torch.float32, (rows,))
    if R is not None:
        _need(R, "R", torch.float32, (rows, K))
    check("int8_rotate_quantize_rows",
          load().int8_rotate_quantize_rows(_ptr(X), rows, K, int(G), _ptr(Xq), _ptr(absmax),
                                           _ptr(R) if R is not None else None, _stream(stream)))
    return Xq, absmax


def int8_rotated_workspace_size(M: int, N: int, K: int) -> int:
    return int(load().int8_rotated_workspace_size(M, N, K))


def int8_rotated_matmul(X, Wq, w_scale, G=128, Y=None, workspace=None, stream=None):
    """W8A8 after grouped Hadamard rotation; returns (Y fp16 [M, N], workspace)."""
    M, K = X.shape
    N = Wq.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq, "Wq", torch.int8, (N, K))
    _need(w_scale, "w_scale", torch.float32, (N,))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int8_rotated_workspace_size(M, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int8_rotated_matmul",
          load().int8_rotated_matmul(_ptr(X), _ptr(Wq), _ptr(w_scale), M, N, K, int(G), _ptr(Y),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)))
    return Y, workspace


def rotated_workspace_views(workspace: torch.Tensor, M: int, K: int) -> dict:
    """status / x_scale / Xq views of an int8_rotated_matmul workspace."""
    def up(x):
        return (x + 255) // 256 * 256
    xs = up(16)
    xq = up(xs + 4 * M)
    return {"status": workspace[0:4].view(torch.int32),
            "x_scale": workspace[xs:xs + 4 * M].view(torch.float32),
            "Xq": workspace[xq:xq + M * K].view(torch.int8).view(M, K)}


def int4_rotate_quantize_groups(X, G=128, Xq=True, Xp=True, absmax=None, stream=None):
    """Rotate, per-(row, group) absmax, 4-bit codes. Xq / Xp: True to allocate,
    None to skip, or a tensor (int8 [rows, K] / int32 [rows, K/8] holding the
    packed uint32 words). Returns (Xq or None, Xp or None, absmax fp32 [rows, K/G])."""
    rows, K = X.shape
    _need(X, "X", torch.float16, (rows, K))
    if Xq is True:
        Xq = torch.empty((rows, K), dtype=torch.int8, device=X.device)
    if Xp is True:
        Xp = torch.empty((rows, K // 8), dtype=torch.int32, device=X.device)
    if absmax is None:
        absmax = torch.empty((rows, K // max(int(G), 1)), dtype=torch.float32, device=X.device)
    if Xq is not None:
        _need(Xq, "Xq", torch.int8, (rows, K))
    if Xp is not None:
        _need(Xp, "Xp", torch.int32, (rows, K // 8))
    check("int4_rotate_quantize_groups",
          load().int4_rotate_quantize_groups(_ptr(X), rows, K, int(G),
                                             _ptr(Xq) if Xq is not None else None,
                                             _ptr(Xp) if Xp is not None else None,
                                             _ptr(absmax), _stream(stream)))
    return Xq, Xp, absmax


def int4_rotate_quantize_weight_blocks(W, G=128, Wp=None, absmax=None, stream=None):
    """Offline W4 weight: rotate rows, per G x G block absmax, packed codes.
    Returns (Wp int32 [N, K/8] holding uint32 words, absmax fp32 [N/G, K/G])."""
    N, K = W.shape
    _need(W, "W", torch.float16, (N, K))
    Wp = torch.empty((N, K // 8), dtype=torch.int32, device=W.device) if Wp is None else Wp
    if absmax is None:
        absmax = torch.empty((max(N // int(G), 0), K // int(G)), dtype=torch.float32,
                             device=W.device)
    _need(Wp, "Wp", torch.int32, (N, K // 8))
    check("int4_rotate_quantize_weight_blocks",
          load().int4_rotate_quantize_weight_blocks(_ptr(W), N, K, int(G), _ptr(Wp), _ptr(absmax),
                                                    _stream(stream)))
    return Wp, absmax


def int4_unpack(P, K, Q=None, stream=None):
    """Packed 4-bit codes int32 [rows, K/8] (uint32 words) -> int8 [rows, K]."""
    rows = P.shape[0]
    _need(P, "P", torch.int32, (rows, K // 8))
    Q = torch.empty((rows, K), dtype=torch.int8, device=P.device) if Q is None else Q
    _need(Q, "Q", torch.int8, (rows, K))
    check("int4_unpack", load().int4_unpack(_ptr(P), rows, K, _ptr(Q), _stream(stream)))
    return Q


def int4_rotated_workspace_size(M: int, N: int, K: int, G: int) -> int:
    return int(load().int4_rotated_workspace_size(M, N, K, G))


def int4_rotated_matmul(X, Wq4, w_absmax, G=128, Y=None, workspace=None, stream=None):
    """W4A4 after grouped Hadamard rotation; Wq4 int8 [N, K] holds the weight's
    4-bit codes one per byte, w_absmax fp32 [N/G, K/G]. Returns (Y, workspace)."""
    M, K = X.shape
    N = Wq4.shape[0]
    _need(X, "X", torch.float16, (M, K))
    _need(Wq4, "Wq4", torch.int8, (N, K))
    _need(w_absmax, "w_absmax", torch.float32, (N // int(G), K // int(G)))
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _need(Y, "Y", torch.float16, (M, N))
    need = int4_rotated_workspace_size(M, N, K, G)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    check("int4_rotated_matmul",
          load().int4_rotated_matmul(_ptr(X), _ptr(Wq4), _ptr(w_absmax), M, N, K, int(G), _ptr(Y),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)))
    return Y, workspace


def int4_rotated_workspace_views(workspace: torch.Tensor, M: int, K: int, G: int) -> dict:
    """status / x_absmax / Xq views of an int4_rotated_matmul workspace."""
    def up(x):
        return (x + 255) // 256 * 256
    xa = up(16)
    xq = up(xa + 4 * M * (K // G))
    return {"status": workspace[0:4].view(torch.int32),
            "x_absmax": workspace[xa:xa + 4 * M * (K // G)].view(torch.float32).view(M, K // G),
            "Xq": workspace[xq:xq + M * K].view(torch.int8).view(M, K)}


def selftest_wait_timeout(stream=None) -> int:
    """Runs the bounded-wait self-test; returns the status the device recorded
    (I8MM_ERR_TIMEOUT when the wait gave up as designed). Takes about 2 s."""
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    check("int8_selftest_wait_timeout",
          load().int8_selftest_wait_timeout(_ptr(status), _stream(stream)))
    torch.cuda.synchronize()
    return int(status.item())
