"""Grouped Hadamard rotation on the GPU against the oracle (developer.baidu.com
grouped-rotation article, sections 2, 5.1, 5.2, 5.4).

The rotated fp32 values, the INT8 / 4-bit codes, the packed words and every
absmax are compared bit for bit (the rotation's float64 butterfly sums are exact,
so both sides round the same number); Y within the Y tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_quantized_matmul_b200 as m

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 1e-2, 1e-3


def _y_close(Y, Yref):
    Y = Y.astype(np.float64)
    Yref = Yref.astype(np.float64)
    d = np.abs(Y - Yref)
    assert d.max() <= MAX_REL * np.abs(Yref).max()
    assert d.mean() <= MEAN_REL * np.abs(Yref).mean()


def _wide_range(rows, K, seed):
    """fp16 values over a wide dynamic range (exactness of the sums matters)."""
    rs = np.random.default_rng(seed)
    x = rs.standard_normal((rows, K)) * np.exp2(rs.integers(-18, 12, (rows, K)))
    return np.clip(x, -60000, 60000).astype(np.float16)


ROW_CASES = [(37, 256, 16), (300, 4096, 128), (8, 1024, 256), (65, 1536, 64), (3, 32768, 128),
             (5, 16384, 32), (1, 16, 16)]


@pytest.mark.parametrize("case", ROW_CASES, ids=[f"r{c[0]}-K{c[1]}-G{c[2]}" for c in ROW_CASES])
def test_rotate_rows_bit_exact(case):
    rows, K, G = case
    X = _wide_range(rows, K, seed=rows + K + G) if K <= 4096 else \
        synth.random_case(rows, K, 8, 4, seed=rows + K)[0]
    X[0, :] = 0                                  # an all-zero row: scale 0, codes 0
    q_ref, a_ref, r_ref = oracle.quantize_rows_rotated(X, G)
    Xd = torch.from_numpy(X).cuda()
    R = torch.empty((rows, K), dtype=torch.float32, device="cuda")
    Xq, a = m.int8_rotate_quantize_rows(Xd, G, R=R)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(R.cpu().numpy().view(np.uint32), r_ref.view(np.uint32))
    np.testing.assert_array_equal(a.cpu().numpy(), a_ref)
    np.testing.assert_array_equal(Xq.cpu().numpy(), q_ref)


MM_CASES = [(64, 512, 256, 128, 4), (300, 1040, 136, 16, 3), (129, 4096, 264, 256, 6),
            (16, 4096, 512, 64, 6)]


@pytest.mark.parametrize("case", MM_CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}-G{c[3]}" for c in MM_CASES])
def test_rotated_matmul_parity(case):
    M, K, N, G, n_out = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=M * 3 + K + N + G)
    Wq_ref, aw_ref, _ = oracle.quantize_rows_rotated(W, G)
    ref = oracle.rotated_w8a8_matmul(X, Wq_ref, aw_ref, G)
    Wq, aw = m.int8_rotate_quantize_rows(torch.from_numpy(W).cuda(), G)
    np.testing.assert_array_equal(Wq.cpu().numpy(), Wq_ref)
    np.testing.assert_array_equal(aw.cpu().numpy(), aw_ref)
    Y, work = m.int8_rotated_matmul(torch.from_numpy(X).cuda(), Wq, aw, G)
    torch.cuda.synchronize()
    v = m.rotated_workspace_views(work, M, K)
    assert int(v["status"].item()) == 0
    np.testing.assert_array_equal(v["x_scale"].cpu().numpy(), ref["x_scale"])
    np.testing.assert_array_equal(v["Xq"].cpu().numpy(), ref["Xq"])
    _y_close(Y.cpu().numpy(), ref["Y"])


def test_rotated_matmul_full_size_sampled():
    """The default prefill shape (2048 tokens, K 4096, N 16384): every code and
    scale, and Y on 64 sampled rows."""
    w = synth.WORKLOADS["opt-6.7b-ffn-up-prefill"]
    X, W, _ = synth.make_workload(w)
    G = 128
    Wq_ref, aw_ref, _ = oracle.quantize_rows_rotated(W, G)
    Xq_ref, ax_ref, _ = oracle.quantize_rows_rotated(X, G)
    Wq, aw = m.int8_rotate_quantize_rows(torch.from_numpy(W).cuda(), G)
    Y, work = m.int8_rotated_matmul(torch.from_numpy(X).cuda(), Wq, aw, G)
    torch.cuda.synchronize()
    v = m.rotated_workspace_views(work, w.M, w.K)
    assert int(v["status"].item()) == 0
    np.testing.assert_array_equal(Wq.cpu().numpy(), Wq_ref)
    np.testing.assert_array_equal(aw.cpu().numpy(), aw_ref)
    np.testing.assert_array_equal(v["Xq"].cpu().numpy(), Xq_ref)
    np.testing.assert_array_equal(v["x_scale"].cpu().numpy(), ax_ref)
    rows = np.random.default_rng(5).choice(w.M, 64, replace=False)
    C = oracle.int32_gemm(Xq_ref[rows], Wq_ref)
    Yref = (C.astype(np.float64) * ax_ref[rows].astype(np.float64)[:, None]
            * aw_ref.astype(np.float64)[None, :] / 127.0 ** 2).astype(np.float16)
    _y_close(Y.cpu().numpy()[rows], Yref)


GROUP_CASES = [(37, 256, 16), (300, 4096, 128), (8, 1024, 256), (65, 1536, 64), (4, 32768, 128)]


@pytest.mark.parametrize("case", GROUP_CASES, ids=[f"r{c[0]}-K{c[1]}-G{c[2]}" for c in GROUP_CASES])
def test_int4_groups_bit_exact(case):
    rows, K, G = case
    X = _wide_range(rows, K, seed=7 * rows + K + G)
    X[0, :G] = 0                                 # an all-zero group
    q_ref, a_ref, _ = oracle.quantize_act_groups(X, G)
    Xq, Xp, a = m.int4_rotate_quantize_groups(torch.from_numpy(X).cuda(), G)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a.cpu().numpy(), a_ref)
    np.testing.assert_array_equal(Xq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(Xp.cpu().numpy().view(np.uint32), oracle.pack_int4(q_ref))
    # packed-only call writes the same words
    _, Xp2, a2 = m.int4_rotate_quantize_groups(torch.from_numpy(X).cuda(), G, Xq=None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Xp2.cpu().numpy(), Xp.cpu().numpy())


BLOCK_CASES = [(128, 512, 128), (256, 4096, 128), (64, 1024, 16), (512, 768, 256)]


@pytest.mark.parametrize("case", BLOCK_CASES, ids=[f"N{c[0]}-K{c[1]}-G{c[2]}" for c in BLOCK_CASES])
def test_int4_weight_blocks_bit_exact(case):
    N, K, G = case
    W = synth.make_weight(N, K, 0.02, seed=N + K + G)
    W[:G, :G] = 0                                # an all-zero block
    q_ref, a_ref, _ = oracle.quantize_weight_blocks(W, G)
    Wp, a = m.int4_rotate_quantize_weight_blocks(torch.from_numpy(W).cuda(), G)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a.cpu().numpy(), a_ref)
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32), oracle.pack_int4(q_ref))


def test_empty_rows_and_bad_group():
    X = torch.zeros((0, 256), dtype=torch.float16, device="cuda")
    Xq, a = m.int8_rotate_quantize_rows(X, 128)
    assert Xq.shape == (0, 256) and a.shape == (0,)
    with pytest.raises(m.Int8mmError):
        m.int8_rotate_quantize_rows(torch.zeros((2, 96), dtype=torch.float16, device="cuda"), 64)


def test_int4_unpack_bit_exact():
    rs = np.random.default_rng(3)
    q = rs.integers(-8, 8, (37, 512)).astype(np.int8)
    P = torch.from_numpy(oracle.pack_int4(q).view(np.int32)).cuda()
    Q = m.int4_unpack(P, 512)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Q.cpu().numpy(), q)


W4_CASES = [(64, 512, 256, 128), (300, 1024, 384, 64), (129, 4096, 512, 256), (16, 4096, 1024, 128),
            (2048, 1024, 4096, 128), (1, 256, 64, 64)]


@pytest.mark.parametrize("case", W4_CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}-G{c[3]}" for c in W4_CASES])
def test_int4_rotated_matmul_parity(case):
    """Codes and group maxima bit for bit; Y of the group-scaled tensor-core GEMM
    within the Y tolerance of the oracle's float64 sum over groups."""
    M, K, N, G = case
    X, W, _ = synth.random_case(M, K, N, 6, seed=M + 5 * K + N + G)
    Wq_ref, aw_ref, _ = oracle.quantize_weight_blocks(W, G)
    ref = oracle.rotated_w4a4_matmul(X, oracle.pack_int4(Wq_ref), aw_ref, G)
    Wp, aw = m.int4_rotate_quantize_weight_blocks(torch.from_numpy(W).cuda(), G)
    Wq4 = m.int4_unpack(Wp, K)
    Y, work = m.int4_rotated_matmul(torch.from_numpy(X).cuda(), Wq4, aw, G)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Wq4.cpu().numpy(), Wq_ref)
    np.testing.assert_array_equal(aw.cpu().numpy(), aw_ref)
    v = m.int4_rotated_workspace_views(work, M, K, G)
    assert int(v["status"].item()) == 0
    np.testing.assert_array_equal(v["x_absmax"].cpu().numpy(), ref["x_scale"])
    np.testing.assert_array_equal(v["Xq"].cpu().numpy(), ref["Xq"])
    _y_close(Y.cpu().numpy(), ref["Y"])


def test_exact_half_integer_quotients_round_to_even():
    """Groups of G = 64 with two spikes v1 = 255 + 2k, v2 = 253 - 2k rotate to
    (v1 + v2)/8 = 63.5 (the row absmax) and (v1 - v2)/8, so the odd columns'
    quotient r * 127 / a is exactly k + 1/2: the code path's near-tie fallback
    must give the ties-to-even integer. Same for the 4-bit grid with
    v1 = 15 + 2k, v2 = 13 - 2k (quotient k + 1/2 of r * 7 / a)."""
    G = 64
    ks = np.arange(0, 127)
    X = np.zeros((1, G * len(ks)), np.float16)
    for i, k in enumerate(ks):
        X[0, G * i] = 255 + 2 * k
        X[0, G * i + 1] = 253 - 2 * k
    q_ref, a_ref, _ = oracle.quantize_rows_rotated(X, G)
    assert a_ref[0] == 63.5
    Xq, a = m.int8_rotate_quantize_rows(torch.from_numpy(X).cuda(), G)
    q = Xq.cpu().numpy()
    np.testing.assert_array_equal(q, q_ref)
    even = np.where(ks % 2 == 0, ks, ks + 1)            # rint(k + 1/2), ties to even
    np.testing.assert_array_equal(q[0, G * np.arange(len(ks)) + 1], even)

    ks4 = np.arange(0, 7)
    X4 = np.zeros((1, G * len(ks4)), np.float16)
    for i, k in enumerate(ks4):
        X4[0, G * i] = 15 + 2 * k
        X4[0, G * i + 1] = 13 - 2 * k
    q4_ref, a4_ref, _ = oracle.quantize_act_groups(X4, G)
    Xq4, _, a4 = m.int4_rotate_quantize_groups(torch.from_numpy(X4).cuda(), G, Xp=None)
    q4 = Xq4.cpu().numpy()
    np.testing.assert_array_equal(q4, q4_ref)
    np.testing.assert_array_equal(a4.cpu().numpy(), a4_ref)
    even4 = np.where(ks4 % 2 == 0, ks4, ks4 + 1)
    np.testing.assert_array_equal(q4[0, G * np.arange(len(ks4)) + 1], even4)
