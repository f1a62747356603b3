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


def _apply_cuda(X_local, Wq, w_scale, W_fp16, bitmaps, Y=None, workspace=None):
    return _ops.int8_mixed_matmul_sharded(X_local, Wq, w_scale, W_fp16, bitmaps, Y=Y,
                                          workspace=workspace)[0]


def token_sharded_mixed_matmul(X_local, Wq, w_scale, W_fp16, threshold=6.0, group=None, Y=None,
                               workspace=None, *, find=_find_cuda, gather=_gather,
                               apply=_apply_cuda):
    """This rank's rows of Y for a batch whose tokens are split over `group`."""
    bitmap = find(X_local, threshold)
    bitmaps = gather(bitmap, group)
    return apply(X_local, Wq, w_scale, W_fp16, bitmaps, Y, workspace)
