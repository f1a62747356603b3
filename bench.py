"""Benchmark of the LLM.int8() mixed-precision matmul on B200.

One step = one int8_mixed_matmul call (outlier detection, per-token INT8
quantisation with outlier compaction, tcgen05 INT8 GEMM + fp16 outlier product
+ dequantising epilogue) over one batch of synthetic activations, with the
weight already quantised (int8_quantize_weight_rows runs once, untimed, as
a deployed layer would). The default workload is the largest single-GPU
configuration, the Llama-70B-like FFN prefill (4096 x 8192 . 28672 x 8192);
the same line carries the OPT-6.7B prefill, the outlier-density stress shapes,
the decode shape and the next rows as extra objects.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): by default (--dp sharded) each rank
holds its own tokens of one batch of N*M tokens; the ranks all-gather their
outlier bitmaps once per step so that every rank quantises against the same
outlier set. --dp replicas runs independent full replicas instead. The timed
region is bracketed by barriers, the time is the max over ranks and `value`
counts the work of all ranks ("scaling": "weak").

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "int8_mixed_matmul TOPS & % of B200 INT8 peak; decode-shape HBM GB/s"
DEFAULT_WORKLOAD = "llama-70b-ffn-prefill"
OPT_WORKLOAD = "opt-6.7b-ffn-up-prefill"
DECODE_WORKLOAD = "decode"
STRESS_WORKLOADS = ["stress-o0", "stress-o7", "stress-o64", "stress-o256", "stress-thr-inf",
                    "stress-thr-0"]
# Fallback denominators when MEASURED_PEAKS.json is absent (earlier pool measurement).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Dense INT8 : dense BF16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s nominal).
INT8_OVER_BF16 = 2.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clock_samples(lines)


def summarize_clock_samples(lines):
    """Median SM clock, max clock, throttle reasons seen and peak power from
    `nvidia-smi --format=csv,noheader,nounits` lines of ClockSampler.FIELDS."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

    def num(x):
        return x.replace(".", "", 1).isdigit()

    sm = [float(r[1]) for r in rows if num(r[1])]
    smax = [float(r[2]) for r in rows if num(r[2])]
    pw = [float(r[3]) for r in rows if num(r[3])]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": reasons, "samples": len(rows),
            "power_w_max": max(pw) if pw else None}


# --------------------------------------------------------------------------- oracle timing
def oracle_sample_step(X, W, Wq, w_scale, threshold, rows):
    """The CPU oracle on a `rows`-token batch of the workload (detection over that batch)."""
    import oracle
    Xs = X[:rows]
    return oracle.llm_int8_matmul(Xs, W, threshold, Wq=Wq, w_scale=w_scale, intermediates=False)


def time_oracle(w, X, W, Wq, w_scale, budget_s: float, max_rows: int | None = None):
    """Times the oracle on a bounded row sample of about budget_s seconds.

    The row count is grown from a 16-row probe until one sample takes about the
    budget (the first calls carry fixed costs, so the estimate is refined up to
    three times); when the whole workload fits in the budget, the full step is
    repeated until the budget is spent. Returns (TOPS, rows, seconds per step,
    steps timed)."""
    cap = w.M if max_rows is None else min(w.M, max_rows)
    rows = min(cap, 16)
    t = 0.0
    for _ in range(4):
        t0 = time.perf_counter()
        oracle_sample_step(X, W, Wq, w_scale, w.threshold, rows)
        t = time.perf_counter() - t0
        if t >= 0.5 * budget_s or rows >= cap:
            break
        rows = min(cap, max(rows + 1, int(rows * budget_s / max(t, 1e-6))))
    steps, total = 1, t
    while rows >= cap and total + t <= budget_s and steps < 8:
        t0 = time.perf_counter()
        oracle_sample_step(X, W, Wq, w_scale, w.threshold, rows)
        total += time.perf_counter() - t0
        steps += 1
    t = total / steps
    return 2.0 * rows * w.N * w.K / t / 1e12, rows, t, steps


# --------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int, want_pg: bool = False):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 or (want_pg and "MASTER_ADDR" in os.environ):
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    import torch.distributed as dist
    if ws > 1 or (dist.is_available() and dist.is_initialized()):
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- our arm
class Problem:
    """Device buffers for one workload, replicated into rotating sets."""

    def __init__(self, w, X, W, n_sets):
        import torch
        import w8a8_quantized_matmul_b200 as m
        self.w = w
        Xd = torch.from_numpy(X).cuda()
        Wd = torch.from_numpy(W).cuda()
        Wq, ws = m.int8_quantize_weight_rows(Wd)       # offline, untimed
        Wt = m.int8_transpose_weight(Wd)                # offline: the [K][N] fp16 weight
        del Wd
        need = m.int8_mixed_matmul_workspace_size(w.M, w.N, w.K)
        self.sets = []
        for i in range(n_sets):
            s = dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq if i == 0 else Wq.clone(),
                     ws=ws if i == 0 else ws.clone(), W=Wt if i == 0 else Wt.clone(),
                     Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                     work=torch.empty((need,), dtype=torch.uint8, device="cuda"))
            self.sets.append(s)
        torch.cuda.synchronize()

    def step(self, i):
        import w8a8_quantized_matmul_b200 as m
        s = self.sets[i % len(self.sets)]
        if self.sharded:
            self.sharded_step(s)
            return
        m.int8_mixed_matmul(s["X"], s["Wq"], s["ws"], s["W"], self.w.threshold, Y=s["Y"],
                            workspace=s["work"])

    sharded = False

    def enable_sharding(self, world):
        """Token-sharded steps: this rank's tokens, outlier bitmaps all-gathered."""
        import torch
        words = (self.w.K + 31) // 32
        for s in self.sets:
            s["bm"] = torch.empty((words,), dtype=torch.int32, device="cuda")
            s["cnt"] = torch.empty((4,), dtype=torch.int32, device="cuda")
            s["idx"] = torch.empty((self.w.K,), dtype=torch.int32, device="cuda")
            s["gathered"] = torch.empty((world, words), dtype=torch.int32, device="cuda")
        self.sharded = True

    def sharded_step(self, s):
        import torch.distributed as dist
        import w8a8_quantized_matmul_b200 as m
        m.int8_find_outlier_cols(s["X"], self.w.threshold, col_bitmap=s["bm"],
                                 n_outliers=s["cnt"][:1], col_idx=s["idx"])
        dist.all_gather_into_tensor(s["gathered"], s["bm"])
        m.int8_mixed_matmul_sharded(s["X"], s["Wq"], s["ws"], s["W"], s["gathered"], Y=s["Y"],
                                    workspace=s["work"])

    def time_stage(self, stage, n, stream):
        """Average device time of one stage launched n times back to back (ms)."""
        import torch
        import w8a8_quantized_matmul_b200 as m
        for i in range(3):
            s = self.sets[i % len(self.sets)]
            m.int8_mixed_matmul_stage(stage, s["X"], s["Wq"], s["ws"], s["W"], self.w.threshold,
                                      s["Y"], s["work"])
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(n):
            s = self.sets[i % len(self.sets)]
            m.int8_mixed_matmul_stage(stage, s["X"], s["Wq"], s["ws"], s["W"], self.w.threshold,
                                      s["Y"], s["work"])
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def time_stage_graph(self, stage, n, stream):
        """Average device time of one stage from a CUDA graph of back-to-back
        launches cycling through the rotating sets (ms): the launch rate of the
        host does not enter, as it does for a stage shorter than one Python call."""
        import torch
        import w8a8_quantized_matmul_b200 as m
        per_graph = len(self.sets) * max(1, 32 // len(self.sets))

        def launches():
            for i in range(per_graph):
                s = self.sets[i % len(self.sets)]
                m.int8_mixed_matmul_stage(stage, s["X"], s["Wq"], s["ws"], s["W"],
                                          self.w.threshold, s["Y"], s["work"])

        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            launches()                        # warm the capture stream
            with torch.cuda.graph(g, stream=cap):
                launches()
        torch.cuda.current_stream().wait_stream(cap)
        for _ in range(2):
            g.replay()
        replays = max(3, n // per_graph)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(replays):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / (replays * per_graph)

    def bytes_touched(self):
        w = self.w
        return 2 * w.M * w.K + w.M * w.K + w.N * w.K + 2 * w.M * w.N


def n_sets_for(w, l2_bytes):
    per = 2 * w.M * w.K + w.M * w.K + w.N * w.K + 2 * w.M * w.N
    return int(min(32, max(2, math.ceil(2 * l2_bytes / per) + 1)))


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of each kernel as it is now, keyed by kernel and workload; the
# summaries and their commands are in profiles/. A kernel changed since its
# capture has no entry (its traffic is reported as null).
NCU_TRAFFIC = {
    ("gemm", "llama-70b-ffn-prefill"): {
        "bytes": 371393280 + 217390848,
        "source": "profiles/gemm_i8_persistent_llama-70b-ffn-prefill.md"},
    ("quantize", "llama-70b-ffn-prefill"): {
        "bytes": 68038144 + 5652736,
        "source": "profiles/stream_quantize_llama-70b-ffn-prefill.md"},
    ("quantize", "opt-6.7b-ffn-up-prefill"): {
        "bytes": 17046784 + 0,
        "source": "profiles/stream_quantize_opt-6.7b-ffn-up-prefill.md"},
    ("gemm", "opt-6.7b-ffn-up-prefill"): {
        "bytes": 80.357632e6 + 37.069568e6,
        "source": "profiles/gemm_i8_persistent_opt-6.7b-ffn-up-prefill.md"},
    ("rotate", "opt-6.7b-ffn-up-prefill"): {
        "bytes": 16.804608e6, "source": "profiles/rotate_rows_opt-6.7b-ffn-up-prefill.md"},
    ("decode", "decode"): {
        "bytes": 17029376 + 0, "source": "profiles/decode_kernel_decode-16x4096x4096.md"},
}


def traffic(kernel, workload):
    e = NCU_TRAFFIC.get((kernel, workload))
    return (e["bytes"], e["source"]) if e else (None, None)


def quantize_stage_bytes(w, count):
    """Algorithmic bytes of detection + quantisation (+ compaction) per call."""
    b = 2 * w.M * w.K + w.M * w.K + 4 * w.M     # read X once; write Xq and x_scale
    if count > 0:
        # X_O and W_O written zero-padded to 16 columns; W_O comes from the
        # count contiguous rows of the transposed fp16 weight (2N bytes each).
        pad = (count + 15) // 16 * 16
        b += 2 * w.M * pad + 2 * count * w.N + 2 * w.N * pad
    return b


def timed_loop(fn, n, stream):
    """Average device time (ms) of n back-to-back calls fn(i), CUDA events on `stream`."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(n):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


class Peaks:
    def __init__(self):
        self.d, self.kind = load_peaks()
        self.bf16 = self.d.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        self.bf16_sus = self.d.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        self.int8 = self.bf16 * INT8_OVER_BF16
        self.int8_sus = self.bf16_sus * INT8_OVER_BF16
        self.hbm = self.d.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])


def measure_prefill(w, args, stream, l2, pk, X=None, W=None, steps=None):
    """One prefill workload: whole steps back to back, then each stage alone.

    Returns the object the JSON line carries for it: ms per step and TOPS of the
    whole call, and per stage (quantisation kernel against HBM, GEMM against the
    dense INT8 peak, or the FP16 peak when every column is an outlier)."""
    import w8a8_quantized_matmul_b200 as m
    if X is None:
        X, W, _ = synth.make_workload(w)
    prob = Problem(w, X, W, n_sets_for(w, l2))
    for i in range(max(3, args.warmup)):
        prob.step(i)
    n = steps or max(20, min(args.steps, 200))
    ms = timed_loop(prob.step, n, stream)
    count = int(m.workspace_views(prob.sets[0]["work"], w.M, w.N, w.K)["n_outliers"].item())
    q_ms = prob.time_stage_graph(1, n, stream)
    g_ms = prob.time_stage(2, n, stream)
    ops = 2.0 * w.M * w.N * w.K
    fp16 = count == w.K
    peak = pk.bf16 if fp16 else pk.int8
    qb = quantize_stage_bytes(w, count)
    gt = ops / (g_ms / 1e3) / 1e12
    del prob
    return {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "threshold": w.threshold,
            "detected_outliers": count, "ms_per_step": ms,
            "value": round(ops / (ms / 1e3) / 1e12, 2), "unit": "TOPS",
            "frac_of_peak": round(ops / (ms / 1e3) / 1e12 / peak, 4),
            "peak": ("fp16 dense = measured bf16 burst" if fp16 else "int8 dense = 2 x measured bf16 burst"),
            "gemm": {"ms": g_ms, "achieved": round(gt, 2), "frac": round(gt / peak, 4),
                     "traffic": traffic("gemm", w.name)[0]},
            "quantize": {"ms": q_ms, "achieved_gbs": round(qb / (q_ms / 1e3) / 1e9, 1),
                         "algorithmic_bytes": qb, "frac_of_hbm": round(qb / (q_ms / 1e3) / 1e9 / pk.hbm, 4),
                         "traffic": traffic("quantize", w.name)[0]},
            "calls_timed": n}


def run_ours(args, ws, rank, local):
    import torch
    import w8a8_quantized_matmul_b200 as m
    from w8a8_quantized_matmul_b200 import build as _b
    if rank == 0:
        _b.build()
    barrier(ws)
    m.load()
    pk = Peaks()
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20

    import torch.distributed as dist
    sharded = args.dp == "sharded" and dist.is_available() and dist.is_initialized()
    w = synth.WORKLOADS[args.workload]
    if sharded:
        # this rank's tokens of a batch of ws*M tokens
        X, W, planted = synth.make_workload_shard(w, rank, ws)
    else:
        X, W, planted = synth.make_workload(w)
    n_sets = n_sets_for(w, l2)
    prob = Problem(w, X, W, n_sets)
    if sharded:
        prob.enable_sharding(ws)

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        prob.step(i)
    torch.cuda.synchronize()
    views = m.workspace_views(prob.sets[0]["work"], w.M, w.N, w.K)
    count = int(views["n_outliers"].item())

    # ---- timed region: K steps, barrier + sync on both sides
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        prob.step(i)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, ws)

    # ---- per-kernel times: each stage launched back to back on the same stream
    # (stage 1 = detection/quantisation kernel, stage 2 = GEMM), over the same
    # rotating buffer sets, bracketed by CUDA events.
    n_stage = max(20, min(args.steps, 500))
    q_ms = prob.time_stage_graph(1, n_stage, stream)
    g_ms = prob.time_stage(2, n_stage, stream)
    ops_per_step = 2.0 * w.M * w.N * w.K
    value = ops_per_step * args.steps * ws / (ms_max / 1e3) / 1e12
    gemm_tops = ops_per_step / (g_ms / 1e3) / 1e12
    qbytes = quantize_stage_bytes(w, count)
    q_gbs = qbytes / (q_ms / 1e3) / 1e9

    # ---- the GEMM stage sustained: back to back for a few seconds under the
    # power cap, against the sustained peak, with its own clock record
    sus_n = max(20, int(args.sustain_s * 1e3 / max(g_ms, 1e-3)))
    sclk = ClockSampler(local)
    sclk.start()
    time.sleep(0.2)
    g_sus_ms = prob.time_stage(2, sus_n, stream)
    sus_clk = sclk.stop()
    sus_tops = ops_per_step / (g_sus_ms / 1e3) / 1e12

    # ---- end to end through the public API with host buffers. Every step copies
    # its X in from pinned host memory and its Y back out; the copies run on two
    # copy streams so that step i+1's input and step i-1's output move while step i
    # computes (the rotating device sets are the double buffers; a set is reused
    # only after its previous output has left).
    e2e_steps = min(args.steps, 200)
    Xh = torch.from_numpy(X).pin_memory()
    Yh = torch.empty((w.M, w.N), dtype=torch.float16).pin_memory()
    nsets = len(prob.sets)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nsets)]
    ev_comp = [torch.cuda.Event() for _ in range(nsets)]
    ev_out = [torch.cuda.Event() for _ in range(nsets)]

    def e2e_run(n):
        for i in range(n):
            b = i % nsets
            s = prob.sets[b]
            if i >= nsets:
                s_in.wait_event(ev_comp[b])          # the set's previous X has been read
            with torch.cuda.stream(s_in):
                s["X"].copy_(Xh, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= nsets:
                stream.wait_event(ev_out[b])         # the set's previous Y has left
            prob.step(i)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                Yh.copy_(s["Y"], non_blocking=True)
            ev_out[b].record(s_out)
        for b in range(min(n, nsets)):
            stream.wait_event(ev_out[b])

    e2e_run(nsets)
    torch.cuda.synchronize()
    barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws)
    e2e_value = ops_per_step * e2e_steps * ws / (e2e_ms / 1e3) / 1e12
    del prob, Xh, Yh
    torch.cuda.empty_cache()

    g_traffic, g_src = traffic("gemm", w.name)
    q_traffic, q_src = traffic("quantize", w.name)
    result = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TOPS",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "threshold": w.threshold,
                   "planted_outliers": int(len(planted)), "detected_outliers": count,
                   "parallelism": (f"token-sharded dp{ws}: {ws}x{w.M} tokens per step, one "
                                   "all-gather of the ceil(K/32)-word outlier bitmaps" if sharded
                                   else f"replicas x{ws}"),
                   "l2": f"rotating {n_sets} buffer sets of {prob_bytes(w) / 1e6:.0f} MB "
                         f"touched per step (> 2x L2 of {l2 / 1e6:.0f} MB)"},
        "roofline": {"kernel": "gemm_i8_persistent_kernel (tcgen05 kind::i8 + kind::f16 outlier panels)",
                     "bound": "tensor", "achieved": round(gemm_tops, 2),
                     "peak": round(pk.int8, 1), "unit": "TOPS",
                     "frac": round(gemm_tops / pk.int8, 4),
                     "traffic": g_traffic, "traffic_source": g_src,
                     "peak_note": f"{pk.kind} bf16 burst {pk.bf16} TFLOP/s x {INT8_OVER_BF16} "
                                  "(dense int8 : bf16 nominal ratio)",
                     "gemm_ms": g_ms,
                     "timing": f"{n_stage} back-to-back launches of the GEMM stage, CUDA events",
                     "sustained": {"achieved": round(sus_tops, 2), "peak": round(pk.int8_sus, 1),
                                   "frac_sustained": round(sus_tops / pk.int8_sus, 4),
                                   "gemm_ms": g_sus_ms, "launches": sus_n,
                                   "seconds": round(g_sus_ms * sus_n / 1e3, 2),
                                   "peak_note": f"{pk.kind} bf16 sustained {pk.bf16_sus} TFLOP/s x "
                                                f"{INT8_OVER_BF16}",
                                   "clocks": sus_clk}},
        "roofline_quantize": {"kernel": "stream_quantize_kernel (cooperative, one pass over X)",
                              "bound": "hbm", "achieved": round(q_gbs, 1), "peak": pk.hbm,
                              "unit": "GB/s", "frac": round(q_gbs / pk.hbm, 4),
                              "algorithmic_bytes": qbytes, "stage_ms": q_ms,
                              "timing": "CUDA-graph replay of back-to-back quantisation stages "
                                        "(control-word memset + kernel), CUDA events",
                              "traffic": q_traffic, "traffic_source": q_src,
                              "peak_note": f"{pk.kind} hbm_gbs"},
        "e2e": {"value": round(e2e_value, 3), "unit": "TOPS", "steps": e2e_steps,
                "h2d_bytes_per_step": 2 * w.M * w.K, "d2h_bytes_per_step": 2 * w.M * w.N,
                "pipelining": "copy-in, call and copy-out of consecutive steps on three streams "
                              "(rotating device sets as double buffers)"},
        "gpu_launches": (3 if sharded else 2) * args.steps,
        "gpu_launches_note": ("per step: detect_outliers_kernel (this rank's tokens), the "
                              "quantisation kernel with the gathered bitmaps, the GEMM kernel "
                              "(plus cudaMemsetAsync and the NCCL all-gather)" if sharded else
                              "per step: stream_quantize_kernel and the GEMM kernel "
                              "(plus one cudaMemsetAsync of the control words)"),
        "clocks": clk,
    }
    extras = w.name == DEFAULT_WORKLOAD and not args.no_extras and not sharded
    if extras:
        result["opt"] = measure_prefill(synth.WORKLOADS[OPT_WORKLOAD], args, stream, l2, pk)
        result["stress"] = [measure_prefill(synth.WORKLOADS[n], args, stream, l2, pk)
                            for n in STRESS_WORKLOADS]
    if w.name != DECODE_WORKLOAD and not args.no_extras:
        result["decode"] = bench_decode(args, stream, l2, pk.hbm)
    if extras:
        result["smoothquant"] = bench_smoothquant(args, stream, l2, pk.int8, pk.hbm)
        result["topk"] = [bench_topk(args, stream, l2, pk.int8, f) for f in (0.01, 0.02)]
        result["zeropoint"] = bench_zeropoint(args, stream, l2, pk.int8)
        result["rotation"] = bench_rotation(args, stream, l2, pk.int8, pk.hbm)
        result["rotation_w4a4"] = bench_w4a4(args, stream, l2, pk.int8)
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        Wq_o, ws_o = oracle.quantize_weight_rows(W)
        tops, rows, t, n = time_oracle(w, X, W, Wq_o, ws_o, budget_s=args.cpu_budget)
        result["cpu_baseline"] = {"value": round(tops, 6), "unit": "TOPS",
                                  "cores": oracle.threads(), "kind": "oracle",
                                  "oracle": "C++17 (oracle/llm_int8.cpp), std::thread over rows",
                                  "cpu": cpu_model(),
                                  "sample": f"{rows} of {w.M} tokens of the same workload "
                                            f"(detection over those tokens), {t:.2f} s per "
                                            f"sample, mean of {n}"}
    return result


def prob_bytes(w):
    return 2 * w.M * w.K + w.M * w.K + w.N * w.K + 2 * w.M * w.N


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def bench_decode(args, stream, l2, hbm):
    """Decode shape (16 tokens): HBM GB/s of one int8_mixed_matmul call.

    The kernel is timed from a CUDA graph of back-to-back calls (device time per
    call, as a decode loop that replays graphs sees it); the eager Python loop is
    reported beside it as the host-bound rate of one un-captured call."""
    import torch
    w = synth.WORKLOADS[DECODE_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    n_sets = n_sets_for(w, l2)
    prob = Problem(w, X, W, n_sets)
    for i in range(max(3, args.warmup)):
        prob.step(i)
    steps = max(50, min(args.steps, 2000))
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for i in range(steps):
        prob.step(i)
    e.record(stream)
    torch.cuda.synchronize()
    eager_ms = s.elapsed_time(e) / steps
    # Graph of per_graph calls cycling through the rotating sets (inputs > L2 per cycle).
    per_graph = n_sets * max(1, 64 // n_sets)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for i in range(per_graph):            # warm the capture stream
            prob.step(i)
        with torch.cuda.graph(g, stream=cap):
            for i in range(per_graph):
                prob.step(i)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(3):
        g.replay()
    replays = max(3, steps // per_graph)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(replays):
        g.replay()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / (replays * per_graph)
    del g
    # Algorithmic bytes: read Wq, w_scale, X; write Y (the outlier columns of W are tiny).
    nbytes = w.N * w.K + 4 * w.N + 2 * w.M * w.K + 2 * w.M * w.N
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "us_per_call": round(ms * 1e3, 2),
            "value": round(gbs, 1), "unit": "GB/s", "frac_of_hbm": round(gbs / hbm, 4),
            "algorithmic_bytes": nbytes, "traffic": traffic("decode", w.name)[0],
            "traffic_source": traffic("decode", w.name)[1], "rotating_sets": n_sets,
            "calls_timed": replays * per_graph, "timing": "cuda-graph replay",
            "eager_us_per_call": round(eager_ms * 1e3, 2)}


def bench_smoothquant(args, stream, l2, int8_peak, hbm):
    """SmoothQuant W8A8 on the default prefill shape: calibration, smoothing and the
    weight side once (offline), then the runtime call (smooth + quantise kernel,
    INT8 GEMM) timed back to back over rotating buffers."""
    import torch
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[OPT_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    act = m.int8_column_absmax(Xd)             # calibration on this batch, as the pages do
    wmax = m.int8_column_absmax(Wd)
    s, r = m.int8_smoothquant_factors(act, wmax, 0.5)
    Wq, ws = m.int8_smoothquant_weight_rows(Wd, s)
    n_sets = n_sets_for(w, l2)
    need = m.int8_smoothquant_workspace_size(w.M, w.N, w.K)
    sets = [dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq if i == 0 else Wq.clone(),
                 ws=ws, r=r, Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                 work=torch.empty((need,), dtype=torch.uint8, device="cuda"))
            for i in range(n_sets)]

    def step(i):
        st = sets[i % n_sets]
        m.int8_smoothquant_matmul(st["X"], st["Wq"], st["ws"], st["r"], Y=st["Y"],
                                  workspace=st["work"])

    for i in range(max(3, args.warmup)):
        step(i)
    steps = max(20, min(args.steps, 500))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    tops = 2.0 * w.M * w.N * w.K / (ms / 1e3) / 1e12
    del sets
    return {"workload": w.name, "alpha": 0.5, "ms_per_call": ms, "value": round(tops, 2),
            "unit": "TOPS", "frac_of_int8_peak": round(tops / int8_peak, 4), "steps": steps,
            "rotating_sets": n_sets,
            "kernels": "smooth_quantize_kernel + gemm_i8_persistent_kernel (no outlier pass)"}


def bench_topk(args, stream, l2, int8_peak, fraction):
    """Top-k decomposition on the default prefill shape: the k = round(fraction*K)
    columns of largest max |x| in FP16, timed back to back over rotating buffers."""
    import torch
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[OPT_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Wt = m.int8_transpose_weight(Wd)                    # offline: the [K][N] fp16 weight
    k = int(round(fraction * w.K))
    n_sets = n_sets_for(w, l2)
    need = int(m.load().int8_mixed_matmul_topk_workspace_size(w.M, w.N, w.K))
    sets = [dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq if i == 0 else Wq.clone(), ws=ws,
                 W=Wt if i == 0 else Wt.clone(),
                 Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                 work=torch.empty((need,), dtype=torch.uint8, device="cuda"))
            for i in range(n_sets)]

    def step(i):
        st = sets[i % n_sets]
        m.int8_mixed_matmul_topk(st["X"], st["Wq"], st["ws"], st["W"], k, Y=st["Y"],
                                 workspace=st["work"])

    for i in range(max(3, args.warmup)):
        step(i)
    steps = max(20, min(args.steps, 500))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    tops = 2.0 * w.M * w.N * w.K / (ms / 1e3) / 1e12
    del sets
    return {"workload": w.name, "fraction": fraction, "k": k, "ms_per_call": ms,
            "value": round(tops, 2), "unit": "TOPS", "frac_of_int8_peak": round(tops / int8_peak, 4),
            "steps": steps, "rotating_sets": n_sets,
            "kernels": "column max, top-k select, quantisation with the selected set, GEMM "
                       "(outlier product on the tensor cores for k > 16)"}


def bench_zeropoint(args, stream, l2, int8_peak):
    """The decomposition with zero-point codes on the default prefill shape, timed
    back to back over rotating buffers (weight row sums computed once, offline)."""
    import torch
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[OPT_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wq, ws = m.int8_quantize_weight_rows(Wd)
    Wt = m.int8_transpose_weight(Wd)                    # offline: the [K][N] fp16 weight
    rsum = m.int8_weight_rowsum(Wq)
    n_sets = n_sets_for(w, l2)
    need = int(m.load().int8_mixed_matmul_zp_workspace_size(w.M, w.N, w.K))
    sets = [dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq if i == 0 else Wq.clone(), ws=ws,
                 W=Wt if i == 0 else Wt.clone(),
                 Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                 work=torch.empty((need,), dtype=torch.uint8, device="cuda"))
            for i in range(n_sets)]

    def step(i):
        st = sets[i % n_sets]
        m.int8_mixed_matmul_zp(st["X"], st["Wq"], st["ws"], rsum, st["W"], w.threshold,
                               Y=st["Y"], workspace=st["work"])

    for i in range(max(3, args.warmup)):
        step(i)
    steps = max(20, min(args.steps, 500))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    tops = 2.0 * w.M * w.N * w.K / (ms / 1e3) / 1e12
    del sets
    return {"workload": w.name, "threshold": w.threshold, "ms_per_call": ms,
            "value": round(tops, 2), "unit": "TOPS", "frac_of_int8_peak": round(tops / int8_peak, 4),
            "steps": steps, "rotating_sets": n_sets,
            "kernels": "detect_quantize_compact_kernel<., zero-point> + "
                       "gemm_i8_persistent_kernel<., ., zero-point>"}


def bench_rotation(args, stream, l2, int8_peak, hbm, G=128):
    """W8A8 after grouped Hadamard rotation on the default prefill shape: the weight
    rotated and quantised once (offline), then the runtime call (rotation +
    per-token quantisation kernel, INT8 GEMM) timed back to back over rotating
    buffers; the rotation kernel is also timed alone (its HBM roofline)."""
    import torch
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[OPT_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wq, ws = m.int8_rotate_quantize_rows(Wd, G)
    n_sets = n_sets_for(w, l2)
    need = m.int8_rotated_workspace_size(w.M, w.N, w.K)
    sets = [dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq if i == 0 else Wq.clone(), ws=ws,
                 Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                 work=torch.empty((need,), dtype=torch.uint8, device="cuda"),
                 q=torch.empty((w.M, w.K), dtype=torch.int8, device="cuda"),
                 a=torch.empty((w.M,), dtype=torch.float32, device="cuda"))
            for i in range(n_sets)]

    def step(i):
        st = sets[i % n_sets]
        m.int8_rotated_matmul(st["X"], st["Wq"], st["ws"], G, Y=st["Y"], workspace=st["work"])

    def rot(i):
        st = sets[i % n_sets]
        m.int8_rotate_quantize_rows(st["X"], G, Xq=st["q"], absmax=st["a"])

    def timed(fn, steps):
        for i in range(max(3, args.warmup)):
            fn(i)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(steps):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    steps = max(20, min(args.steps, 500))
    ms = timed(step, steps)
    r_ms = timed(rot, steps)
    tops = 2.0 * w.M * w.N * w.K / (ms / 1e3) / 1e12
    rbytes = 2 * w.M * w.K + w.M * w.K + 4 * w.M
    r_gbs = rbytes / (r_ms / 1e3) / 1e9
    del sets
    return {"workload": w.name, "group": G, "ms_per_call": ms, "value": round(tops, 2),
            "unit": "TOPS", "frac_of_int8_peak": round(tops / int8_peak, 4), "steps": steps,
            "rotating_sets": n_sets,
            "kernels": "rotate_rows_kernel + gemm_i8_persistent_kernel (no outlier pass)",
            "rotate_kernel": {"ms": r_ms, "achieved": round(r_gbs, 1), "unit": "GB/s",
                              "peak": hbm, "frac": round(r_gbs / hbm, 4),
                              "algorithmic_bytes": rbytes,
                              "bytes_note": "X fp16 read + codes written + scales",
                              "traffic": (traffic("rotate", w.name)[0] if G == 128 else None),
                              "traffic_source": traffic("rotate", w.name)[1]}}


def bench_w4a4(args, stream, l2, int8_peak, G=128):
    """W4A4 after grouped Hadamard rotation on the default prefill shape: the weight
    rotated, block-quantised, packed and expanded to one code per byte once
    (offline), then the runtime call (rotation + per-(token, group) 4-bit codes,
    group-scaled tensor-core GEMM) timed back to back over rotating buffers."""
    import torch
    import w8a8_quantized_matmul_b200 as m
    w = synth.WORKLOADS[OPT_WORKLOAD]
    X, W, _ = synth.make_workload(w)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    Wp, aw = m.int4_rotate_quantize_weight_blocks(Wd, G)
    Wq4 = m.int4_unpack(Wp, w.K)
    del Wd
    n_sets = n_sets_for(w, l2)
    need = m.int4_rotated_workspace_size(w.M, w.N, w.K, G)
    sets = [dict(X=Xd if i == 0 else Xd.clone(), Wq=Wq4 if i == 0 else Wq4.clone(),
                 Y=torch.empty((w.M, w.N), dtype=torch.float16, device="cuda"),
                 work=torch.empty((need,), dtype=torch.uint8, device="cuda"))
            for i in range(n_sets)]

    def step(i):
        st = sets[i % n_sets]
        m.int4_rotated_matmul(st["X"], st["Wq"], aw, G, Y=st["Y"], workspace=st["work"])

    for i in range(max(3, args.warmup)):
        step(i)
    steps = max(20, min(args.steps, 500))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    tops = 2.0 * w.M * w.N * w.K / (ms / 1e3) / 1e12
    del sets
    return {"workload": w.name, "group": G, "ms_per_call": ms, "value": round(tops, 2),
            "unit": "TOPS", "frac_of_int8_peak": round(tops / int8_peak, 4), "steps": steps,
            "rotating_sets": n_sets,
            "kernels": "rotate_groups_kernel + gemm_groups_kernel (4-bit codes on the INT8 "
                       "tensor cores, per-group promotion)",
            "weight_bytes_packed": w.N * w.K // 2}


# --------------------------------------------------------------------------- reference arm
def run_reference(args, ws, rank):
    """The CPU oracle as the reference arm, on bounded samples of the same workload."""
    import oracle
    w = synth.WORKLOADS[args.workload]
    X, W, _ = synth.make_workload(w)
    Wq, w_scale = oracle.quantize_weight_rows(W)
    total = args.steps + args.warmup
    per_step_budget = max(0.02, args.ref_budget / max(total, 1))
    rows = min(w.M, 16)
    t0 = time.perf_counter()
    oracle_sample_step(X, W, Wq, w_scale, w.threshold, rows)
    t1 = time.perf_counter() - t0
    rows = max(1, min(w.M, int(rows * per_step_budget / max(t1, 1e-6))))
    for _ in range(args.warmup):
        oracle_sample_step(X, W, Wq, w_scale, w.threshold, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(X, W, Wq, w_scale, w.threshold, rows)
    t = time.perf_counter() - t0
    tops = 2.0 * rows * w.N * w.K * args.steps / t / 1e12
    cores = oracle.threads()
    sample = f"{rows} of {w.M} tokens per step (detection over those tokens)"
    return {
        "impl": "reference", "metric": METRIC, "value": round(tops, 6), "unit": "TOPS",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "threshold": w.threshold},
        "cpu_baseline": {"value": round(tops, 6), "unit": "TOPS", "cores": cores,
                         "kind": "oracle", "oracle": "C++17 (oracle/llm_int8.cpp), std::thread over rows",
                         "cpu": cpu_model(), "sample": sample},
        "e2e": {"value": round(tops, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work in all steps of --impl reference together")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the chosen workload (no OPT, stress, decode and next-row objects)")
    ap.add_argument("--sustain-s", type=float, default=2.5,
                    help="seconds of back-to-back GEMM launches for the sustained figure")
    ap.add_argument("--dp", default="sharded", choices=["sharded", "replicas"],
                    help="with several ranks: split the tokens of one batch over the ranks "
                         "(one all-gather of the outlier bitmaps per step) or run full replicas")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, ws, rank)), flush=True)
        return

    ws, rank, local = dist_setup(args.gpus, want_pg=(args.dp == "sharded"))
    try:
        res = run_ours(args, ws, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
