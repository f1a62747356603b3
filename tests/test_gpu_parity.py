"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer and byte outputs (outlier bitmap, count, ascending column list,
INT8 codes, absmax scales, INT32 accumulators, compacted panels) must match
bit for bit. The fp16 Y must satisfy, against the oracle's Y,
    max|dY| <= 1e-2 * max|Y_ref|   and   mean|dY| <= 1e-3 * mean|Y_ref|.
Both sides take every integer decision (|x| > threshold, rint of the fp32
quotient) in fp32, so the codes can be compared exactly.
"""
import math
import zlib

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_TOL = 1e-2
MEAN_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_quantized_matmul_b200 import build
    build.build()


def mm():
    import w8a8_quantized_matmul_b200 as m
    return m


def wt(W):
    """The fp16 weight in the transposed [K][N] layout the mixed-matmul calls take."""
    return mm().int8_transpose_weight(W)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def assert_y_close(Y, Yref, what=""):
    Y = np.asarray(Y, np.float64)
    Yref = np.asarray(Yref, np.float64)
    assert np.all(np.isfinite(Y)), f"{what}: non-finite output"
    d = np.abs(Y - Yref)
    r = np.abs(Yref)
    assert d.max() <= MAX_TOL * r.max() + 1e-6, f"{what}: max|dY|={d.max()} max|Y|={r.max()}"
    assert d.mean() <= MEAN_TOL * r.mean() + 1e-7, f"{what}: mean|dY|={d.mean()} mean|Y|={r.mean()}"


def run_mixed(X, W, thr):
    """Runs the whole path on the GPU; returns (Y, workspace views as numpy, Wq, w_scale)."""
    m = mm()
    Xd, Wd = dev(X), dev(W)
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y, work = m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), thr)
    views = m.workspace_views(work, X.shape[0], W.shape[0], X.shape[1])
    out = {k: host(v) for k, v in views.items()}
    assert m.int8_device_status(work) == 0
    return host(Y), out, host(Wq), host(ws)


def check_intermediates(ref, got, K):
    count = ref["count"]
    assert int(got["n_outliers"][0]) == count
    assert np.array_equal(got["col_bitmap"].view(np.uint32), ref["bitmap"])
    assert np.array_equal(got["col_idx"][:count], ref["idx"])
    assert np.array_equal(got["Xq"], ref["Xq"])
    assert np.array_equal(got["x_scale"].view(np.uint32), ref["x_scale"].view(np.uint32))


def check_panels(X, W, ref, got):
    """Compacted fp16 outlier panels, zero-padded to a multiple of 16 columns
    (one kind::f16 K step; the GEMM multiplies only the steps that hold columns)."""
    count = ref["count"]
    if count == 0 or X.shape[0] <= 16:   # no panels (or the decode path)
        return
    pad = (count + 15) // 16 * 16
    idx = ref["idx"]
    assert np.array_equal(got["X_O"][:, :count], X[:, idx])
    assert np.all(got["X_O"][:, count:pad] == 0)
    assert np.array_equal(got["W_O"][:, :count], W[:, idx])
    assert np.all(got["W_O"][:, count:pad] == 0)


# ---------------------------------------------------------------- weight quant
@pytest.mark.parametrize("N,K", [(256, 256), (264, 272), (8, 16), (33, 48), (3, 12288), (129, 4096)])
def test_quantize_weight_rows_bitexact(N, K):
    W = synth.make_weight(N, K, 0.02, seed=N + K)
    W[min(2, N - 1), :] = 0
    Wq, ws = mm().int8_quantize_weight_rows(dev(W))
    rq, rs = oracle.quantize_weight_rows(W)
    assert np.array_equal(host(Wq), rq)
    assert np.array_equal(host(ws).view(np.uint32), rs.view(np.uint32))


# ---------------------------------------------------------------- weight layout
@pytest.mark.parametrize("N,K", [(256, 256), (33, 48), (1, 16), (129, 4096), (70000, 16), (8, 12288)])
def test_transpose_weight_exact(N, K):
    """int8_transpose_weight gives W^T element for element (ragged tiles included)."""
    W = synth.make_weight(N, K, 0.02, seed=N * 3 + K)
    Wt = mm().int8_transpose_weight(dev(W))
    assert tuple(Wt.shape) == (K, N)
    assert np.array_equal(host(Wt).view(np.uint16), np.ascontiguousarray(W.T).view(np.uint16))


# ---------------------------------------------------------------- detection
@pytest.mark.parametrize("M,K,n_out,thr", [(16, 256, 2, 6.0), (200, 272, 5, 6.0), (1, 16, 1, 6.0),
                                           (33, 4096, 7, 6.0), (64, 1040, 40, 6.0), (70, 512, 3, math.inf),
                                           (70, 512, 3, 0.0), (40, 1024, 9, 30.0), (0, 64, 0, 6.0)])
def test_find_outlier_cols_bitexact(M, K, n_out, thr):
    X, _, _ = synth.random_case(max(M, 1), K, 8, n_out, seed=M * 7 + K)
    X = X[:M]
    if M > 3:
        X[0, K // 2] = np.float16(6.0)          # equal to the threshold
        X[:, 3] = 0                               # all-zero column
    bm, cnt, idx = mm().int8_find_outlier_cols(dev(X) if M else torch.empty((0, K), dtype=torch.float16, device="cuda"), thr)
    _, rbm, rc, ridx = oracle.find_outlier_cols(X, thr)
    assert int(host(cnt)[0]) == rc
    assert np.array_equal(host(bm).view(np.uint32), rbm)
    assert np.array_equal(host(idx)[:rc], ridx)


# ---------------------------------------------------------------- activation quant
@pytest.mark.parametrize("M,K,n_out", [(16, 256, 2), (200, 272, 5), (1, 16, 0), (9, 8192, 7),
                                       (5, 12288, 3), (300, 4096, 64), (3, 2048, 0)])
def test_quantize_act_rows_bitexact(M, K, n_out):
    X, _, _ = synth.random_case(M, K, 8, n_out, seed=M + 3 * K)
    if M > 2:
        X[1, :] = 0                               # all-zero row
        a = 127.0 / 64.0                          # rounding ties: 32.5 -> 32, 33.5 -> 34
        X[2, :] = 0
        X[2, :4] = np.array([a, 65 / 128, 67 / 128, -65 / 128], np.float16)
    mask, bitmap, _, _ = oracle.find_outlier_cols(X, 6.0)
    Xq, xs = mm().int8_quantize_act_rows(dev(X), dev(bitmap.view(np.int32)))
    rq, rs = oracle.quantize_act_rows(X, mask)
    assert np.array_equal(host(Xq), rq)
    assert np.array_equal(host(xs).view(np.uint32), rs.view(np.uint32))
    if M > 2 and not mask[:4].any():
        assert host(Xq)[2, :4].tolist() == [127, 32, 34, -32]


# ---------------------------------------------------------------- INT32 GEMM
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 264, 272), (1, 8, 16), (300, 520, 1040),
                                   (129, 257, 4096), (16, 4096, 512)])
def test_debug_gemm_i32_bitexact(M, N, K):
    rs = np.random.default_rng(M * N + K)
    Xq = rs.integers(-127, 128, size=(M, K)).astype(np.int8)
    Wq = rs.integers(-127, 128, size=(N, K)).astype(np.int8)
    C = mm().int8_debug_gemm_i32(dev(Xq), dev(Wq))
    assert np.array_equal(host(C), oracle.int32_gemm(Xq, Wq))


def test_debug_gemm_i32_overflow_bound():
    K = 8192
    Xq = np.full((130, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.full((260, K), 127, np.int8)
    C = host(mm().int8_debug_gemm_i32(dev(Xq), dev(Wq)))
    assert np.all(C[0] == 127 * 127 * K) and np.all(C[1] == -127 * 127 * K)
    assert np.array_equal(C, oracle.int32_gemm(Xq, Wq))


# ---------------------------------------------------------------- full path
MIXED_CASES = [
    # name, M, K, N, n_outliers, threshold
    ("tiny-workload", None, None, None, None, None),
    ("ragged", 200, 272, 264, 3, 6.0),
    ("no-outliers", 130, 512, 256, 0, 6.0),
    ("seven", 256, 1024, 512, 7, 6.0),
    ("64-outliers", 256, 1024, 512, 64, 6.0),
    ("65-outliers", 129, 1024, 260, 65, 6.0),
    ("130-outliers", 257, 2048, 384, 130, 6.0),
    ("thr-inf", 256, 1024, 512, 7, math.inf),
    ("thr-0", 200, 512, 264, 7, 0.0),
    ("single-token", 1, 4096, 512, 3, 6.0),
    ("decode-17", 17, 4096, 1024, 6, 6.0),
    ("narrow-N", 64, 256, 8, 2, 6.0),
    ("K16", 40, 16, 40, 1, 6.0),
    ("K48-N-odd", 40, 48, 37, 1, 6.0),
]


@pytest.mark.parametrize("case", MIXED_CASES, ids=[c[0] for c in MIXED_CASES])
def test_mixed_matmul_parity(case):
    name, M, K, N, n_out, thr = case
    if name == "tiny-workload":
        w = synth.WORKLOADS["tiny"]
        X, W, _ = synth.make_workload(w)
        thr = w.threshold
    else:
        X, W, _ = synth.random_case(M, K, N, n_out, seed=zlib.crc32(name.encode()) % 1000)
        if M > 4:
            X[4, :] = 0                            # all-zero token
    Y, got, Wq, ws = run_mixed(X, W, thr)
    ref = oracle.llm_int8_matmul(X, W, thr)
    assert np.array_equal(Wq, ref["Wq"])
    check_intermediates(ref, got, X.shape[1])
    check_panels(X, W, ref, got)
    assert_y_close(Y, ref["Y"], name)


DECODE_CASES = [
    # M, K, N, n_outliers, threshold
    (1, 4096, 512, 3, 6.0),
    (3, 272, 130, 2, 6.0),
    (16, 1024, 256, 5, 6.0),
    (16, 3072, 520, 6, 6.0),       # three CTAs per cluster, ragged row split
    (16, 8192, 384, 7, 6.0),       # eight CTAs per cluster
    (7, 2048, 8, 4, 6.0),
    (16, 512, 200, 6, math.inf),
    (16, 512, 200, 6, 0.0),        # every nonzero column is an outlier
    (12, 4096, 1000, 0, 6.0),
    (16, 4096, 256, 64, 6.0),      # more outliers per CTA than are gathered ahead
    (5, 1040, 136, 3, 6.0),        # two ranks, the last K-block 16 columns wide
    (8, 12288, 256, 5, 6.0),       # K > 8192: too long for one cluster, the prefill kernels run
    (16, 16384, 136, 7, 6.0),      # the same, 16 tokens, ragged N
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}-o{c[3]}-t{c[4]}" for c in DECODE_CASES])
def test_decode_path_parity(case):
    """Shapes of at most 16 tokens go through the clustered decode kernel (K <= 8192)
    or, for longer rows, through the prefill kernels."""
    M, K, N, n_out, thr = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=M * 1000 + K + N)
    if M > 2:
        X[1, :] = 0
    Y, got, Wq, ws = run_mixed(X, W, thr)
    ref = oracle.llm_int8_matmul(X, W, thr)
    check_intermediates(ref, got, K)
    assert_y_close(Y, ref["Y"], f"decode {case}")


RECHECK_CASES = [
    # M, K, N: the first has more rows per CTA than the kernel's row slots
    (4096, 8192, 256),
    (2048, 4096, 520),
    (300, 1040, 136),
    (37, 4096, 64),
]


@pytest.mark.parametrize("case", RECHECK_CASES, ids=[f"M{c[0]}-K{c[1]}-N{c[2]}" for c in RECHECK_CASES])
def test_outliers_on_few_tokens_force_the_recheck(case):
    """The fused kernel quantises each CTA's rows against the CTA's own outlier
    columns and checks them against the whole batch's afterwards. Outlier columns
    whose outliers sit on one or two tokens are missing from almost every CTA's
    own set, so those CTAs must redo their rows (re-reading them through the
    row slots when they do not all fit); the result must not change."""
    M, K, N = case
    X, W, cols = synth.random_case(M, K, N, 3, seed=M + K + N)
    free = [j for j in range(K) if j not in set(cols.tolist())]
    j1, j2 = free[K // 3], free[2 * K // 3 + 5]
    X[M // 2 + 3, j1] = np.float16(50.0)             # one token only
    X[1, j2] = np.float16(-7.5)                      # two tokens far apart
    X[M - 1, j2] = np.float16(9.0)
    Y, got, Wq, ws = run_mixed(X, W, 6.0)
    ref = oracle.llm_int8_matmul(X, W, 6.0)
    assert ref["count"] == 5
    check_intermediates(ref, got, K)
    check_panels(X, W, ref, got)
    assert_y_close(Y, ref["Y"], f"recheck {case}")


@pytest.mark.parametrize("thr", [6.001, 5.999, 65519.0, 70000.0, 1e-9, 2.0 ** -24, 0.5])
def test_threshold_between_fp16_values(thr):
    """Thresholds that no fp16 value equals (and the neighbours of the ones that
    are): the prefill kernel's fp16 comparison selects the oracle's fp32 set."""
    M, K, N = 96, 512, 136
    X, W, _ = synth.random_case(M, K, N, 4, seed=77)
    t16 = np.float16(thr)
    near = [t16, np.nextafter(t16, np.float16(np.inf)), np.nextafter(t16, np.float16(0))]
    near = [v for v in near if np.isfinite(v)]      # finite inputs only
    for j, v in enumerate(near):                    # entries at and next to the threshold
        X[3 + j, 7 * j + 1] = v
        X[20 + j, 11 * j + 5] = -v
    X[40, 100] = np.float16(65504.0)
    Y, got, _, _ = run_mixed(X, W, thr)
    ref = oracle.llm_int8_matmul(X, W, thr)
    check_intermediates(ref, got, K)
    check_panels(X, W, ref, got)
    assert_y_close(Y, ref["Y"], f"threshold {thr}")


def test_mixed_matmul_guard_bands():
    """Writes stay inside Y and the workspace (256-byte canaries on both sides)."""
    m = mm()
    M, K, N = 131, 272, 264
    X, W, _ = synth.random_case(M, K, N, 3, seed=5)
    Xd, Wd = dev(X), dev(W)
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    G = 256
    ybuf = torch.full((2 * G + M * N * 2,), 0xA5, dtype=torch.uint8, device="cuda")
    Y = ybuf[G:G + M * N * 2].view(torch.float16).view(M, N)
    need = m.int8_mixed_matmul_workspace_size(M, N, K)
    wbuf = torch.full((2 * G + need,), 0x5A, dtype=torch.uint8, device="cuda")
    work = wbuf[G:G + need]
    m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), 6.0, Y=Y, workspace=work)
    yb = host(ybuf)
    wb = host(wbuf)
    assert np.all(yb[:G] == 0xA5) and np.all(yb[G + M * N * 2:] == 0xA5)
    assert np.all(wb[:G] == 0x5A) and np.all(wb[G + need:] == 0x5A)
    assert_y_close(host(Y), oracle.llm_int8_matmul(X, W, 6.0)["Y"], "guarded")


def test_mixed_matmul_repeated_calls_reuse_workspace():
    """A second call with other data on the same workspace gives that data's result."""
    m = mm()
    X1, W, _ = synth.random_case(150, 512, 200, 5, seed=21)
    X2, _, _ = synth.random_case(150, 512, 200, 9, seed=22)
    Wd = dev(W)
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y1, work = m.int8_mixed_matmul(dev(X1), Wq, ws, wt(Wd), 6.0)
    y1 = host(Y1).copy()
    Y2, _ = m.int8_mixed_matmul(dev(X2), Wq, ws, wt(Wd), 6.0, workspace=work)
    assert_y_close(host(Y2), oracle.llm_int8_matmul(X2, W, 6.0)["Y"], "second call")
    assert_y_close(y1, oracle.llm_int8_matmul(X1, W, 6.0)["Y"], "first call")


def test_stage_hook_reproduces_full_call():
    """Stage 1 then stage 2 of the measurement hook give the full call's Y bit for bit."""
    m = mm()
    X, W, _ = synth.random_case(300, 1024, 520, 6, seed=31)
    Xd, Wd = dev(X), dev(W)
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y1, work = m.int8_mixed_matmul(Xd, Wq, ws, wt(Wd), 6.0)
    y1 = host(Y1).copy()
    Y2 = torch.zeros_like(Y1)
    work2 = torch.zeros_like(work)
    m.int8_mixed_matmul_stage(1, Xd, Wq, ws, wt(Wd), 6.0, Y2, work2)
    m.int8_mixed_matmul_stage(2, Xd, Wq, ws, wt(Wd), 6.0, Y2, work2)
    assert np.array_equal(host(Y2), y1)
    m.int8_mixed_matmul_stage(2, Xd, Wq, ws, wt(Wd), 6.0, Y2, work2)   # GEMM alone again
    assert np.array_equal(host(Y2), y1)


def test_empty_problem_is_a_noop():
    m = mm()
    W = dev(synth.make_weight(64, 64, 0.02, seed=1))
    Wq, ws = m.int8_quantize_weight_rows(W)
    X = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    Y, _ = m.int8_mixed_matmul(X, Wq, ws, wt(W), 6.0)
    assert tuple(Y.shape) == (0, 64)


# ---------------------------------------------------------------- every fp16 input value
def _every_value_rows(amaxes):
    """Row i holds amaxes[i] and every finite fp16 x with |x| <= amaxes[i] (zero-padded)."""
    allh = np.arange(65536, dtype=np.uint16).view(np.float16)
    allh = allh[np.isfinite(allh)]
    rows = []
    for a in amaxes:
        a16 = np.float16(a)
        v = allh[np.abs(allh.astype(np.float32)) <= np.float32(a16)]
        rows.append(np.concatenate([[a16], v]))
    K = (max(r.size for r in rows) + 15) // 16 * 16
    X = np.zeros((len(rows), K), np.float16)
    for i, r in enumerate(rows):
        X[i, :r.size] = r
    return X


AMAXES = [127 / 64, 6.0, 5.99609375, 1.0, 0.5, 3.140625, 0.0078125, 2.0 ** -14, 1000.0, 0.333251953125]


def test_quantize_every_fp16_value_standalone():
    """All rounding cases (exact ties, near-ties, clamps) of the quantiser, bit-exact."""
    X = _every_value_rows(AMAXES)
    K = X.shape[1]
    mask = np.zeros(K, bool)
    bitmap = np.zeros((K + 31) // 32, np.uint32)
    Xq, xs = mm().int8_quantize_act_rows(dev(X), dev(bitmap.view(np.int32)))
    rq, rs = oracle.quantize_act_rows(X, mask)
    assert np.array_equal(host(xs), rs)
    assert np.array_equal(host(Xq), rq)


def test_quantize_every_fp16_value_fused_path():
    """The same sweep through int8_mixed_matmul (threshold=inf: no outliers)."""
    X = _every_value_rows(AMAXES[:6])
    K = X.shape[1]
    W = synth.make_weight(8, K, 0.02, seed=77)
    Y, got, Wq, ws = run_mixed(X, W, math.inf)
    ref = oracle.llm_int8_matmul(X, W, math.inf)
    check_intermediates(ref, got, K)
    assert_y_close(Y, ref["Y"], "every-value")
