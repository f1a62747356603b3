"""Token-sharded (data-parallel over tokens) LLM.int8() matmul across ranks.

AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section: the
outlier feature dimensions are the columns where any token of the batch exceeds
the threshold. When a batch's tokens are split over ranks, the ranks must agree
on one set before quantising, which is the one exchange step of this path:

  1. each rank detects on its own rows (int8_find_outlier_cols, its kernel);
  2. the ranks all-gather their bitmaps (ceil(K/32) words each, one collective);
  3. each rank runs int8_mixed_matmul_sharded on its rows with all the bitmaps;
     the kernel ORs them, then quantises and multiplies exactly as the
     single-process path does.

The concatenation of the ranks' Y equals the single-process Y over the whole
batch, element for element. `find`, `gather` and `apply` default to the CUDA
kernels and torch.distributed; they are parameters so that the exchange logic
can be exercised with other implementations of the same three steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

import w8a8_quantized_matmul_b200 as _ops


def _find_cuda(X_local, threshold):
    bitmap, _, _ = _ops.int8_find_outlier_cols(X_local, threshold)
    return bitmap


def _gather(bitmap, group=None):
    """All ranks' bitmaps as one [world, words] int32 tensor, in rank order."""
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world, bitmap.numel()), dtype=bitmap.dtype, device=bitmap.device)
        dist.all_gather_into_tensor(out, bitmap.contiguous(), group=group)
        return out
    parts = [torch.empty_like(bitmap) for _ in range(world)]
    dist.all_gather(parts, bitmap.contiguous(), group=group)
    return torch.stack(parts)


def _apply_cuda(X_local, Wq, w_scale, Wt_fp16, bitmaps, Y=None, workspace=None):
    return _ops.int8_mixed_matmul_sharded(X_local, Wq, w_scale, Wt_fp16, bitmaps, Y=Y,
                                          workspace=workspace)[0]


def token_sharded_mixed_matmul(X_local, Wq, w_scale, Wt_fp16, threshold=6.0, group=None, Y=None,
                               workspace=None, *, find=_find_cuda, gather=_gather,
                               apply=_apply_cuda):
    """This rank's rows of Y for a batch whose tokens are split over `group`."""
    bitmap = find(X_local, threshold)
    bitmaps = gather(bitmap, group)
    return apply(X_local, Wq, w_scale, Wt_fp16, bitmaps, Y, workspace)


# ---------------------------------------------------------------------------
# Column-sharded (out-feature) form. The outlier set is a function of X alone
# (AIInfra "05Quantization01", LLM.int8() section: a feature dimension is an
# outlier when some activation in it exceeds the threshold), so ranks that each
# hold all of X and a contiguous block of the weight's output rows derive the
# same set with no exchange; every output column depends only on its own weight
# row. Each rank's Y is a column block of the whole Y; gathering the blocks is
# needed only if a caller wants the full Y on every rank.
# ---------------------------------------------------------------------------
def column_block(N: int, rank: int, world: int):
    """[n0, n1) of rank's output rows: contiguous blocks, multiples of 8 rows
    where possible (keeps the weight slices' addresses 16-byte aligned)."""
    per = (N + world - 1) // world
    per = (per + 7) // 8 * 8
    n0 = min(N, rank * per)
    return n0, min(N, n0 + per)


def _apply_cols_cuda(X, Wq_local, w_scale_local, Wt_local, threshold, Y=None, workspace=None):
    return _ops.int8_mixed_matmul(X, Wq_local, w_scale_local, Wt_local, threshold, Y=Y,
                                  workspace=workspace)[0]


def _gather_cols(Y_local, N, group=None):
    """The column blocks of all ranks as one [M, N] tensor (blocks in rank order)."""
    world = dist.get_world_size(group)
    per = (N + world - 1) // world
    per = (per + 7) // 8 * 8
    parts = [torch.empty((Y_local.shape[0], per), dtype=Y_local.dtype, device=Y_local.device)
             for _ in range(world)]
    pad = torch.zeros((Y_local.shape[0], per), dtype=Y_local.dtype, device=Y_local.device)
    pad[:, :Y_local.shape[1]] = Y_local
    dist.all_gather(parts, pad, group=group)
    return torch.cat(parts, dim=1)[:, :N]


def column_sharded_mixed_matmul(X, Wq_local, w_scale_local, Wt_local, threshold=6.0, group=None,
                                N=None, gather=False, Y=None, workspace=None, *,
                                apply=_apply_cols_cuda):
    """This rank's column block of Y = X . W^T from its block of weight rows
    (`column_block`: Wq_local and w_scale_local are rows [n0, n1) of Wq and
    w_scale, Wt_local the columns [n0, n1) of the transposed fp16 weight as a
    contiguous [K, n1 - n0] tensor); no collective unless gather=True, which
    returns the full [M, N] Y on every rank (N is then required)."""
    Y_local = apply(X, Wq_local, w_scale_local, Wt_local, threshold, Y, workspace)
    if not gather:
        return Y_local
    if N is None:
        raise ValueError("gather=True needs the full N")
    return _gather_cols(Y_local, N, group)
