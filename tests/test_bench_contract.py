"""The benchmark's command-line contract, on the CPU (no GPU needed).

`bench.py --impl reference` runs the CPU oracle as the reference arm and prints
one JSON line with the keys the driver reads; fewer than 3 warm-up steps are
refused before any work.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e"}


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-budget", "4"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"] == "llama-70b-ffn-prefill"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "C++" in cb["oracle"]
    assert cb["unit"] == d["unit"] and "tokens" in cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_too_few_warmup_steps_refused():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "2"], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 2
    assert "warmup" in r.stderr


def test_clock_samples_summary():
    import bench
    lines = [
        "0, 1965, 1965, 412.50, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1950, 1965, 870.25, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1440, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "garbage line\n",
        "0, [N/A], 1965, [N/A], 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    s = bench.summarize_clock_samples(lines)
    assert s["samples"] == 4
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] == 990.0
    bad = bench.summarize_clock_samples(
        ["0, 900, 1965, 300.0, 0x8, Not Active, Active, Not Active, Not Active\n"])
    assert bad["reasons"] == ["hw_thermal_slowdown"]
    assert bench.summarize_clock_samples([])["samples"] == 0


def test_rotating_sets_exceed_l2():
    import bench
    import synth
    l2 = 126 * 2 ** 20
    for name in ("opt-6.7b-ffn-up-prefill", "decode", "llama-70b-ffn-prefill"):
        w = synth.WORKLOADS[name]
        n = bench.n_sets_for(w, l2)
        per = 2 * w.M * w.K + w.M * w.K + w.N * w.K + 2 * w.M * w.N
        assert n >= 2 and (n * per > 2 * l2 or n == 32)
