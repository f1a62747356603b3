"""Parity at the benchmark's full sizes, in the benchmark's launch configuration.

For every named workload (tiny, OPT-6.7B FFN-up prefill, decode, Llama-70B
FFN prefill, and the outlier-density stress cases with the threshold=inf and
threshold=0 endpoints) the CUDA path runs once through int8_mixed_matmul with
the same workspace layout bench.py uses. Then:
  * the outlier set (bitmap, count, ascending list) and the per-token INT8
    codes and scales of the whole X match the oracle bit for bit;
  * the weight codes and scales match bit for bit;
  * the INT32 accumulators of the tensor-core kernel match exact integer dot
    products at sampled positions;
  * Y matches the oracle, computed one output at a time, at sampled positions
    plus one full row and one full column, within the Y tolerance.
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_TOL = 1e-2
MEAN_TOL = 1e-3
N_SAMPLES = 4096


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_quantized_matmul_b200 import build
    build.build()


def _positions(M, N, seed):
    rs = np.random.default_rng(seed)
    r = rs.integers(0, M, N_SAMPLES)
    c = rs.integers(0, N, N_SAMPLES)
    fr, fc = int(rs.integers(0, M)), int(rs.integers(0, N))
    r = np.concatenate([r, np.full(N, fr), np.arange(M)])
    c = np.concatenate([c, np.arange(N), np.full(M, fc)])
    return r, c


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_workload_parity(name):
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[name]
    X, W, planted = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Y, work = m.int8_mixed_matmul(Xd, Wq, ws, m.int8_transpose_weight(Wd), w.threshold)
    torch.cuda.synchronize()
    assert m.int8_device_status(work) == 0
    views = m.workspace_views(work, w.M, w.N, w.K)

    # Outlier set and activation codes over the whole X.
    mask, bitmap, count, idx = oracle.find_outlier_cols(X, w.threshold)
    if np.isfinite(w.threshold) and w.threshold >= 6.0:
        assert idx.tolist() == planted.tolist()
    assert int(views["n_outliers"].item()) == count
    assert np.array_equal(views["col_bitmap"].cpu().numpy().view(np.uint32), bitmap)
    assert np.array_equal(views["col_idx"][:count].cpu().numpy(), idx)
    Xq_ref, xs_ref = oracle.quantize_act_rows(X, mask)
    assert np.array_equal(views["Xq"].cpu().numpy(), Xq_ref)
    assert np.array_equal(views["x_scale"].cpu().numpy(), xs_ref)

    # Weight codes (all rows).
    Wq_ref, ws_ref = oracle.quantize_weight_rows(W)
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    assert np.array_equal(ws.cpu().numpy(), ws_ref)

    # Y at sampled positions, one output at a time.
    r, c = _positions(w.M, w.N, seed=w.seed)
    Ys, Cs, _, _ = oracle.llm_int8_matmul_at(X, W, Wq_ref, ws_ref, w.threshold, r, c)
    Yg = Y.cpu().numpy()[r, c].astype(np.float64)
    d = np.abs(Yg - Ys.astype(np.float64))
    ref = np.abs(Ys.astype(np.float64))
    assert d.max() <= MAX_TOL * ref.max() + 1e-6, (d.max(), ref.max())
    assert d.mean() <= MEAN_TOL * ref.mean() + 1e-7, (d.mean(), ref.mean())

    # INT32 accumulators of the tensor-core kernel at the same positions.
    C = m.int8_debug_gemm_i32(views["Xq"], Wq)
    torch.cuda.synchronize()
    Cg = C.cpu().numpy()[r, c]
    assert np.array_equal(Cg, Cs)
