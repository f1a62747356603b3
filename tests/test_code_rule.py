"""The division-free INT8 code rule of the CUDA kernels, checked on the CPU.

The kernels replace the one correctly rounded division of the quantiser
(AIInfra "05Quantization01", LLM.int8() section: q = rint(x * 127 / absmax))
by a reciprocal and one FMA correction step. tests/fma_quotient_check.c checks,
for fp16 inputs, that this gives exactly the IEEE quotient and therefore the
same codes, for every pair of positive finite fp16 values x <= absmax (about
5e8 pairs, a few seconds). The check uses no GPU and no code of the CUDA path:
it restates the kernels' arithmetic in plain C.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _build(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "fma_quotient_check")
    subprocess.run([cc, "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                    os.path.join(HERE, "fma_quotient_check.c"), "-lm"], check=True)
    return exe


def _run(exe, stride):
    out = subprocess.run([exe, str(stride)], capture_output=True, text=True, timeout=1800)
    assert out.returncode == 0, out.stdout + out.stderr
    pairs = int(out.stdout.split()[1])
    assert pairs > 0
    return pairs


def test_fma_corrected_quotient_exhaustive(tmp_path):
    # every pair 0 < x <= a of positive finite fp16 values
    assert _run(_build(tmp_path), 1) == 31743 * 31744 // 2
