"""The single-pass quantisation kernel's argument, checked on the CPU.

The kernel codes each row as soon as it is read, with m1 = the row's absmax over
the entries it does not itself flag (|x| > threshold), and only afterwards learns
the batch's outlier set O (AIInfra "05Quantization01", LLM.int8() section: a
column is an outlier when some token exceeds the threshold). Per block of rows
(a CTA) it then zeroes the codes at its own flagged columns L, codes a row again
when its largest entry <= threshold in L reaches m1, and, when the batch's set
has a column the block lacks, codes the whole block again with O. This model
follows those steps in numpy (the code rule itself is the oracle's) and must give
exactly the oracle's codes and scales, including on inputs built so that the
speculation fails. The GPU parity tests check the kernel; this checks the steps."""
import numpy as np
import pytest

import oracle
import synth


def single_pass_model(X, thr, rows_per_block, stats=None):
    a = np.abs(X.astype(np.float32))
    M, K = a.shape
    own = a > np.float32(thr)                                  # entries a row flags itself
    m1 = np.where(own, np.float32(0), a).max(axis=1) if K else np.zeros(M, np.float32)
    codes = oracle.absmax_codes(X.astype(np.float32), m1[:, None], 127).astype(np.int8)
    scale = m1.copy()
    O = own.any(axis=0)
    for r0 in range(0, M, rows_per_block):
        rows = slice(r0, min(M, r0 + rows_per_block))
        L = own[rows].any(axis=0)                               # the block's own set
        blk = a[rows]
        sub = codes[rows]
        sub[:, L] = 0
        codes[rows] = sub
        mO = np.where(L[None, :] & ~own[rows], blk, np.float32(0)).max(axis=1)
        redo = (scale[rows] > 0) & (mO >= scale[rows])
        need = np.nonzero(redo)[0] + r0
        use = O if np.any(O & ~L) else L                        # the batch set when the block lacks a column
        if stats is not None:
            stats["rows"] += len(need)
            stats["blocks"] += int(np.any(O & ~L))
        if np.any(O & ~L):
            need = np.arange(rows.start, rows.stop)
        for r in need:
            keep = ~use
            m = a[r][keep].max() if keep.any() else np.float32(0)
            scale[r] = m
            q = oracle.absmax_codes(X[r].astype(np.float32), m, 127).astype(np.int8)
            q[use] = 0
            codes[r] = q
    return codes, scale, O


def check(X, thr, rows_per_block):
    stats = {"rows": 0, "blocks": 0}
    codes, scale, O = single_pass_model(X, thr, rows_per_block, stats)
    mask, _, _, _ = oracle.find_outlier_cols(X, thr)
    Xq, xs = oracle.quantize_act_rows(X, mask)
    assert np.array_equal(O, mask)
    assert np.array_equal(scale.view(np.uint32), xs.view(np.uint32))
    assert np.array_equal(codes, Xq)
    return stats


@pytest.mark.parametrize("rows_per_block", [1, 3, 7, 64])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_random_batches(rows_per_block, seed):
    X, _, _ = synth.random_case(96, 256, 8, 5, seed=seed)
    check(X, 6.0, rows_per_block)


def test_row_maximum_in_a_column_another_row_flags():
    X, _, cols = synth.random_case(32, 128, 8, 2, seed=9)
    c = int(cols[0])
    X[:, c] = np.float16(0.25)
    X[0, c] = np.float16(40.0)            # row 0 flags column c
    X[5, c] = np.float16(5.5)             # row 5's largest entry sits in c, below the threshold
    X[5, :] = np.clip(X[5, :], -2, 2)
    X[5, c] = np.float16(5.5)
    for rpb in (1, 4, 8, 32):             # row 0 and row 5 in the same block or not
        st = check(X, 6.0, rpb)
        assert st["rows"] + st["blocks"] >= 1   # the speculation failed and was repaired


def test_tie_between_an_outlier_column_and_a_kept_column():
    X, _, cols = synth.random_case(16, 64, 8, 1, seed=4)
    c = int(cols[0])
    X[3, :] = np.float16(0.5)
    X[3, c] = np.float16(3.0)             # in the outlier column
    X[3, (c + 7) % 64] = np.float16(3.0)  # the same value in a kept column
    X[0, c] = np.float16(50.0)
    for rpb in (1, 2, 16):
        st = check(X, 6.0, rpb)
        assert st["rows"] + st["blocks"] >= 1


def test_block_missing_a_column_of_the_batch():
    X, _, _ = synth.random_case(40, 128, 8, 0, seed=12)
    X[37, 11] = np.float16(-9.0)          # only the last block's rows see column 11
    X[2, 11] = np.float16(4.0)            # a large entry of another block in that column
    for rpb in (4, 8):
        assert check(X, 6.0, rpb)["blocks"] >= 1
    check(X, 6.0, 40)


@pytest.mark.parametrize("thr", [0.0, float("inf"), 30.0])
def test_endpoints_and_zero_rows(thr):
    X, _, _ = synth.random_case(24, 64, 8, 3, seed=5)
    X[4, :] = 0
    check(X, thr, 5)
