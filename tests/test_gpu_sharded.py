"""Token-sharded path on one GPU: ranks emulated one after another.

Each "rank" runs int8_find_outlier_cols on its rows; then each runs
int8_mixed_matmul_sharded with every rank's bitmap. The concatenated Y must
equal int8_mixed_matmul over the whole batch element for element (same
outlier set, same per-token scales, exact INT32 products), the intermediates
must equal the oracle's with the batch's outlier set, and the workspace bitmap
must hold the OR ([AIInfra] "05Quantization01", LLM.int8() section).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_quantized_matmul_b200 as m

pytestmark = pytest.mark.gpu


def wt(W):
    """The fp16 weight in the transposed [K][N] layout the mixed-matmul calls take."""
    return m.int8_transpose_weight(W)

CASES = [
    # M, K, N, n_outliers, row bounds of the ranks
    (300, 512, 384, 5, [0, 100, 300]),
    (300, 512, 384, 5, [0, 0, 7, 300]),          # an empty rank, a rank with 7 tokens
    (1024, 4096, 1024, 6, [0, 256, 512, 768, 1024]),
    (256, 1024, 512, 40, [0, 130, 256]),        # 40 outlier columns: one 64-column panel block
]


@pytest.mark.parametrize("case", CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}-o{c[3]}-r{len(c[4]) - 1}" for c in CASES])
def test_sharded_equals_whole_batch(case):
    M, K, N, n_out, bounds = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=M + K + N + len(bounds))
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y_full, _ = m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), 6.0)
    parts = [Xd[bounds[r]:bounds[r + 1]].contiguous() for r in range(len(bounds) - 1)]
    bitmaps = torch.stack([m.int8_find_outlier_cols(p, 6.0)[0] for p in parts])
    ys = []
    ref = oracle.llm_int8_matmul(X, W)
    for r, p in enumerate(parts):
        Y, work = m.int8_mixed_matmul_sharded(p, Wq, ws, wt(Wd), bitmaps)
        ys.append(Y)
        torch.cuda.synchronize()
        if p.shape[0] == 0:
            continue   # nothing launched: the workspace is untouched
        assert m.int8_device_status(work) == 0
        v = m.workspace_views(work, p.shape[0], N, K)
        np.testing.assert_array_equal(v["col_bitmap"].cpu().numpy().view(np.uint32), ref["bitmap"])
        r0, r1 = bounds[r], bounds[r + 1]
        np.testing.assert_array_equal(v["Xq"].cpu().numpy(), ref["Xq"][r0:r1])
        np.testing.assert_array_equal(v["x_scale"].cpu().numpy(), ref["x_scale"][r0:r1])
        assert int(v["n_outliers"].item()) == ref["count"]
    Y_sh = torch.cat(ys, dim=0)
    assert torch.equal(Y_sh, Y_full)
