"""Token-sharded path across processes, on the CPU with the gloo backend.

The exchange logic of w8a8_quantized_matmul_b200.sharded (local detection, one
all-gather of the bitmaps, quantisation and product with their OR) runs with
the CPU oracle standing in for the two kernels. The concatenated rows of Y must
equal the oracle's Y over the whole batch exactly, and the OR of the gathered
bitmaps must equal the whole batch's bitmap ([AIInfra] "05Quantization01",
LLM.int8() section: the outlier set belongs to the batch).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _find(X_local, threshold):
    _, bitmap, _, _ = oracle.find_outlier_cols(X_local.numpy(), threshold)
    return torch.from_numpy(bitmap.view(np.int32).copy())


def _apply(X_local, Wq, w_scale, Wt, bitmaps, Y=None, workspace=None):
    words = bitmaps.numpy().view(np.uint32)
    orw = np.bitwise_or.reduce(words, axis=0)
    K = X_local.shape[1]
    mask = ((orw[np.arange(K) // 32] >> (np.arange(K) % 32).astype(np.uint32)) & 1).astype(bool)
    out = oracle.llm_int8_matmul(X_local.numpy(), np.ascontiguousarray(Wt.numpy().T), Wq=Wq.numpy(),
                                 w_scale=w_scale.numpy(), outlier_mask=mask)
    return torch.from_numpy(out["Y"]), torch.from_numpy(orw.view(np.int32).copy())


def _worker(rank, world, port, bounds, case, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from w8a8_quantized_matmul_b200.sharded import token_sharded_mixed_matmul
        M, K, N, n_out, seed = case
        X, W, _ = synth.random_case(M, K, N, n_out, seed=seed)
        Wq, w_scale = oracle.quantize_weight_rows(W)
        r0, r1 = bounds[rank], bounds[rank + 1]
        Xl = torch.from_numpy(np.ascontiguousarray(X[r0:r1]))
        Y, orw = token_sharded_mixed_matmul(Xl, torch.from_numpy(Wq), torch.from_numpy(w_scale),
                                           torch.from_numpy(np.ascontiguousarray(W.T)), 6.0,
                                           find=_find, apply=_apply)
        q.put((rank, Y.numpy(), orw.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,split", [(2, [0, 37, 96]), (3, [0, 0, 50, 96]), (2, [0, 96, 96])])
def test_token_sharded_matches_whole_batch(world, split):
    case = (96, 320, 72, 4, 11)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, split, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, Y, orw = q.get(timeout=120)
        results[rank] = (Y, orw)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    M, K, N, n_out, seed = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=seed)
    ref = oracle.llm_int8_matmul(X, W)
    Y = np.concatenate([results[r][0] for r in range(world)], axis=0)
    np.testing.assert_array_equal(Y, ref["Y"])
    for r in range(world):
        np.testing.assert_array_equal(results[r][1].view(np.uint32), ref["bitmap"])


def _report_and_exit(q, msg):
    # flush the queue's feeder thread before leaving without the process
    # group's teardown (its peer is gone)
    q.put(msg)
    q.close()
    q.join_thread()
    os._exit(0)


def _failing_worker(rank, world, port, mode, q):
    """Rank 1 leaves (mode "exit") or stalls (mode "stall") before the exchange;
    rank 0 must get an error from its collective instead of waiting forever."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import time
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=3))
        dist.barrier()          # both ranks are up before one of them goes away
    except Exception as e:
        _report_and_exit(q, ("setup failed: " + type(e).__name__, 0.0))
    if rank == 1:
        if mode == "stall":
            time.sleep(12)
        os._exit(0)
    from w8a8_quantized_matmul_b200.sharded import token_sharded_mixed_matmul
    X, W, _ = synth.random_case(16, 64, 8, 1, seed=3)
    Wq, w_scale = oracle.quantize_weight_rows(W)
    t0 = time.perf_counter()
    try:
        token_sharded_mixed_matmul(torch.from_numpy(X), torch.from_numpy(Wq),
                                   torch.from_numpy(w_scale),
                                   torch.from_numpy(np.ascontiguousarray(W.T)), 6.0,
                                   find=_find, apply=_apply)
        msg = ("no error", time.perf_counter() - t0)
    except Exception as e:  # the collective's failure reaches the host as an exception
        msg = (type(e).__name__, time.perf_counter() - t0)
    _report_and_exit(q, msg)


@pytest.mark.parametrize("mode", ["exit", "stall"])
def test_lost_rank_ends_the_exchange_with_an_error(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        what, secs = q.get(timeout=90)
        assert what != "no error" and not what.startswith("setup failed"), what
        assert secs < 30            # the process-group timeout (3 s), not a hang
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()


def _apply_cols(X, Wq_local, w_scale_local, Wt_local, threshold, Y=None, workspace=None):
    out = oracle.llm_int8_matmul(X.numpy(), np.ascontiguousarray(Wt_local.numpy().T), threshold,
                                 Wq=Wq_local.numpy(), w_scale=w_scale_local.numpy())
    return torch.from_numpy(out["Y"])


def _cols_worker(rank, world, port, case, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from w8a8_quantized_matmul_b200.sharded import column_block, column_sharded_mixed_matmul
        M, K, N, n_out, seed = case
        X, W, _ = synth.random_case(M, K, N, n_out, seed=seed)
        n0, n1 = column_block(N, rank, world)
        Wq, w_scale = oracle.quantize_weight_rows(W[n0:n1])
        Y_local = column_sharded_mixed_matmul(torch.from_numpy(X), torch.from_numpy(Wq),
                                              torch.from_numpy(w_scale),
                                              torch.from_numpy(np.ascontiguousarray(W[n0:n1].T)),
                                              6.0, apply=_apply_cols)
        Y_full = column_sharded_mixed_matmul(torch.from_numpy(X), torch.from_numpy(Wq),
                                             torch.from_numpy(w_scale),
                                             torch.from_numpy(np.ascontiguousarray(W[n0:n1].T)),
                                             6.0, N=N, gather=True, apply=_apply_cols)
        q.put((rank, n0, n1, Y_local.numpy(), Y_full.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, (40, 256, 96, 3, 5)), (3, (17, 320, 200, 4, 6))])
def test_column_sharded_matches_whole_layer(world, case):
    """Each rank holds all of X and a block of weight rows: no exchange, the same
    outlier set everywhere, and the column blocks make up the whole Y exactly."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cols_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, n0, n1, Yl, Yf = q.get(timeout=120)
        got[rank] = (n0, n1, Yl, Yf)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    M, K, N, n_out, seed = case
    X, W, _ = synth.random_case(M, K, N, n_out, seed=seed)
    ref = oracle.llm_int8_matmul(X, W)["Y"]
    covered = np.zeros(N, bool)
    for r in range(world):
        n0, n1, Yl, Yf = got[r]
        assert Yl.shape == (M, n1 - n0)
        np.testing.assert_array_equal(Yl, ref[:, n0:n1])
        np.testing.assert_array_equal(Yf, ref)
        covered[n0:n1] = True
    assert covered.all()
